"""gdn_frame_scan_fwd_static: the scan for callers that cannot allocate
device memory per call (a streaming loop that must not stall on cudaMalloc,
memory already held by the host's own pool, a plugin given no workspace).

Runs last (file name) so that a stop at the first failure has already run
every other test. Through the C ABI it checks:
  - the fixed array first holds NaN from a poisoning call, so a later call
    that read a byte it had not written would come out NaN;
  - each plan the entry reaches (chains alongside the contraction in one
    cooperative launch, whose publication counters live in the fixed array;
    the span-composed plan; the token-split contraction), twice in a row,
    against the allocating entry point: bit for bit where the plan is
    deterministic, within the bf16 bound for the token-split plan (its
    partial sums meet in atomic adds, whose order varies);
  - every frame and final state against the float64 oracle (bf16 bound);
  - sizes beyond the fixed 32 MiB are refused before any launch.
"""

import ctypes

import pytest
import torch

from frame_wise_gated_b200 import api
from tests import gdn_testutil as U

pytestmark = pytest.mark.gpu

# (name, B, H, T, S, plan keywords, bit-exact against the allocating entry)
CASES = [
    # one 3-frame block of 16 heads at 720p, reverse with block reset: the
    # streaming use; 48 frame-heads, chains alongside the contraction
    ("overlap_block3_720p", 1, 16, 3, 3600, dict(reverse=True, block_reset=True), True),
    # forward with a start state, 72 frame-heads, ragged last token tile
    ("overlap_fwd_state", 1, 8, 9, 1000, dict(), True),
    # span-composed plan (spans of 8 frames, 2 spans per head)
    ("chunked", 1, 4, 16, 500, dict(chunked=True), True),
    # 6 frame-heads: each frame-head's tokens cut over several CTAs
    ("token_split", 1, 2, 3, 600, dict(), False),
]


def _poison():
    """Fills the part of the fixed array that the largest accepted problem
    uses with NaN-derived values (NaN inputs through both plans)."""
    def fits(T):
        return all(api.workspace_bytes(1, 16, T, 3600, 128, f) <= api.STATIC_SCRATCH_BYTES
                   for f in (api.BF16, api.BF16 | api.CHUNKED))
    T = 1
    while fits(T + 1):
        T += 1
    nan = float("nan")
    q = torch.full((1, 16, T, 3600, 128), nan, device="cuda", dtype=torch.bfloat16)
    beta = torch.full((1, 16, T, 3600), nan, device="cuda")
    gamma = torch.full((1, 16, T), nan, device="cuda")
    state = torch.full((1, 16, 128, 128), nan, device="cuda")
    for kw in (dict(), dict(chunked=True)):
        o, _ = api.frame_scan_fwd_static(q, q, q, beta, gamma, state, **kw)
    torch.cuda.synchronize()
    api.check_device_status()
    assert torch.isnan(o.float()).any()


def _inputs(seed, B, H, T, S):
    arr = U.random_case(seed, B, H, T, S, 128, bf16=True, state=True)
    return arr, U.dev_inputs(arr, True)


def _oracle_error(arr, got_o, got_s, kw):
    B, H = got_o.shape[:2]
    block = 3 if kw.get("block_reset") else 0
    worst = 0.0
    for b in range(B):
        for h in range(H):
            o_ref, s_ref = U.oracle_slab(arr, b, h, True, reverse=kw.get("reverse", False),
                                         block=block)
            worst = max(worst, U.rel_frob_per_frame(U.host(got_o[b, h]), o_ref),
                        U.rel_frob_per_frame(U.host(got_s[b, h])[None], s_ref[None]))
    return worst


def test_static_scratch_matches_allocating_entry_and_oracle():
    _poison()
    for i, (name, B, H, T, S, kw, exact) in enumerate(CASES):
        arr, d = _inputs(80 + i, B, H, T, S)
        ref_o, ref_s = api.frame_scan_fwd(d["q"], d["k"], d["v"], d["beta"], d["gamma"],
                                          d["state"], **kw)
        for call in range(2):  # two calls in a row over the array the last call left
            got_o, got_s = api.frame_scan_fwd_static(d["q"], d["k"], d["v"], d["beta"],
                                                     d["gamma"], d["state"], **kw)
            torch.cuda.synchronize()
            api.check_device_status()
            assert not torch.isnan(got_o.float()).any(), (name, call)
            if exact:
                assert torch.equal(got_o, ref_o), (name, call)
                assert torch.equal(got_s, ref_s), (name, call)
            else:
                assert U.rel_frob_per_frame(U.host(got_o).reshape(-1, S, 128),
                                            U.host(ref_o).reshape(-1, S, 128)) < U.TOL_BF16
            err = _oracle_error(arr, got_o, got_s, kw)
            assert err < U.TOL_BF16, (name, call, err)


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
