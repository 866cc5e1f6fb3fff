"""gdn_frame_scan_fwd_static: the scan for callers that cannot allocate
device memory per call (streaming loops, pool-owned memory, plugin hosts).

Runs last (file name) so that a stop at the first failure has already run
every other test. Checks, through the C ABI, that two calls in a row match
the allocating entry point within the bf16 tolerance of the other tests, and
that sizes beyond the fixed 32 MiB scratch are refused.
"""

import ctypes

import numpy as np
import pytest
import torch

from frame_wise_gated_b200 import api
from tests import gdn_testutil as U

pytestmark = pytest.mark.gpu


def rel(a, b):
    a, b = a.double(), b.double()
    return float((a - b).norm() / b.norm())


def test_static_scratch_matches_allocating_entry_twice():
    cases = [
        dict(seed=71, B=1, H=4, T=6, S=300, D=128, kw=dict()),
        dict(seed=72, B=2, H=3, T=3, S=257, D=128, kw=dict(reverse=True, block_reset=True)),
    ]
    for c in cases:  # two calls in a row, different sizes and contents
        arr = U.random_case(c["seed"], c["B"], c["H"], c["T"], c["S"], c["D"], bf16=True, state=True)
        d = U.dev_inputs(arr, True)
        ref_o, ref_s = api.frame_scan_fwd(d["q"], d["k"], d["v"], d["beta"], d["gamma"],
                                          d["state"], **c["kw"])
        got_o, got_s = api.frame_scan_fwd_static(d["q"], d["k"], d["v"], d["beta"], d["gamma"],
                                                 d["state"], **c["kw"])
        torch.cuda.synchronize()
        api.check_device_status()
        assert rel(got_o.float(), ref_o.float()) < U.TOL_BF16
        assert rel(got_s, ref_s) < U.TOL_BF16


def test_static_scratch_refuses_oversized_problems():
    arr = U.random_case(73, 1, 1, 2, 16, 16, bf16=True)
    d = U.dev_inputs(arr, True)
    L = api.lib()
    # 60 s 720p rollout sizes need far more than 32 MiB: refused before any launch
    rc = L.gdn_frame_scan_fwd_static(*(ctypes.c_void_p(t.data_ptr()) for t in
                                       (d["q"], d["k"], d["v"], d["beta"], d["gamma"])),
                                     None, ctypes.c_void_p(d["q"].data_ptr()), None,
                                     1, 16, 121, 3600, 128, api.BF16, None)
    assert rc == api.GDN_ERR_WORKSPACE
    assert b"32 MiB" in L.gdn_last_error()
