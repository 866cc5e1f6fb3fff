"""B200-native frame-wise Gated DeltaNet (GDN) frame scan.

The compute lives in ``libgdnscan.so`` (hand-written sm_100a CUDA behind a C
ABI declared in ``include/gdn.h``); ``api`` is a thin argument-marshalling
binding over it. ``synth`` draws the seeded synthetic inputs.
"""
