"""Float64 CPU oracle for the frame-wise Gated DeltaNet (GDN) frame scan.

TEST INFRASTRUCTURE ONLY. This package is the slow, plain, obviously correct
statement of what the frame scan computes. Only the test suite, the
``__graft_entry__.smoke`` check and ``bench.py``'s CPU-baseline / reference
legs may import it. The product path (the CUDA library and its Python
binding) never imports, calls or links anything here, and this package never
imports the product path.
"""

from .gdn_oracle import *  # noqa: F401,F403
