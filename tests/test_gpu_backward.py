"""GPU parity of the backward pass (gdn_frame_scan_bwd) against the oracle's
adjoint (pinned by finite differences), through the C ABI.

Metric: per (b, h) slab and per gradient tensor, ||g_gpu - g_ref||_F /
||g_ref||_F; bounds as the forward: 1e-4 for fp32 inputs, 1e-2 for bf16
inputs (the same bf16-rounded inputs and upstream gradients go to the oracle).
"""

import numpy as np
import pytest
import torch

from frame_wise_gated_b200 import api, synth
from oracle import gdn_oracle as O
from tests import gdn_testutil as U

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dbeta", "dgamma", "d_state_in")


def rel(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def upstream(seed, B, H, T, S, D, bf16):
    rng = np.random.default_rng(seed)
    dO = rng.standard_normal((B, H, T, S, D), dtype=np.float32)
    dO = synth.bf16_round_bits(dO) if bf16 else dO
    dS = rng.standard_normal((B, H, D, D)).astype(np.float32)
    return dO, dS


def check_case(arr, dO, dS, bf16, tol, reverse=False, block=0, b_slabs=None, force_simt=False):
    d = U.dev_inputs(arr, bf16)
    d_out = U.to_dev(dO, bf16)
    d_s = torch.from_numpy(dS).cuda() if dS is not None else None
    got = api.frame_scan_bwd(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"], d_out,
                             d_s, reverse=reverse, block_reset=bool(block), block=block or 3,
                             force_simt=force_simt)
    torch.cuda.synchronize()
    api.check_device_status()
    B, H = arr["beta"].shape[:2]
    slabs = b_slabs or [(b, h) for b in range(B) for h in range(H)]
    worst = {}
    for (b, h) in slabs:
        ref = O.frame_scan_bwd(U.widen(arr["q"][b, h], bf16), U.widen(arr["k"][b, h], bf16),
                               U.widen(arr["v"][b, h], bf16), arr["beta"][b, h].astype(np.float64),
                               arr["gamma"][b, h].astype(np.float64),
                               None if arr["state"] is None else arr["state"][b, h],
                               U.widen(dO[b, h], bf16), None if dS is None else dS[b, h],
                               reverse=reverse, block=block)
        for name, g, r in zip(NAMES, got, ref):
            if g is None:
                continue
            e = rel(U.host(g[b, h]), r)
            worst[name] = max(worst.get(name, 0.0), e)
    for name, e in worst.items():
        assert e < tol, (name, e, worst)
    return worst


MODES = {"forward": dict(), "reverse": dict(reverse=True), "forward_block": dict(block=3),
         "reverse_block": dict(reverse=True, block=3)}


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("D,bf16,simt", [(16, False, True), (64, False, True), (128, False, True),
                                         (64, True, True), (128, True, False), (128, True, True),
                                         (256, True, True)])
def test_backward_small(D, bf16, simt, mode):
    """Every mode; D = 128 bf16 on both the tensor-core and the CUDA-core path."""
    B, H, T, S = 2, 1, 7, 150
    arr = U.random_case(3000 + D, B, H, T, S, D, bf16=bf16, state=True)
    dO, dS = upstream(17 + D, B, H, T, S, D, bf16)
    check_case(arr, dO, dS, bf16, U.TOL_BF16 if bf16 else U.TOL_FP32, force_simt=simt,
               **MODES[mode])


def test_backward_many_heads_tc():
    """More heads than chains fit beside the contraction: the recompute runs
    as its own launches (tensor-core path)."""
    arr = U.random_case(51, 1, 40, 4, 70, 128, bf16=True, state=True)
    dO, dS = upstream(52, 1, 40, 4, 70, 128, True)
    check_case(arr, dO, dS, True, U.TOL_BF16, b_slabs=[(0, 0), (0, 17), (0, 39)])


def test_backward_without_state_terms():
    """No state_in, no gradient of state_out: the pure output loss."""
    arr = U.random_case(41, 1, 2, 5, 33, 32, bf16=False, state=False)
    dO, _ = upstream(42, 1, 2, 5, 33, 32, False)
    check_case(arr, dO, None, False, U.TOL_FP32)


def test_backward_edge_sizes():
    for (T, S, D) in [(1, 1, 16), (1, 5, 64), (2, 129, 128), (9, 1, 128)]:
        arr = U.random_case(T * S + D + 7, 1, 1, T, S, D, bf16=True, state=True)
        dO, dS = upstream(T + S + D, 1, 1, T, S, D, True)
        check_case(arr, dO, dS, True, U.TOL_BF16)


def test_backward_three_part_dq_units():
    """Frames of 1496 tokens (12 tiles of 128, the last 88 tokens): the dq
    readout splits each frame-head into three units of 4 tiles."""
    arr = U.random_case(61, 1, 2, 3, 1496, 128, bf16=True, state=True)
    dO, dS = upstream(62, 1, 2, 3, 1496, 128, True)
    check_case(arr, dO, dS, True, U.TOL_BF16)


@pytest.mark.parametrize("name", ["clip5s_720p", "rollout60s_720p"])
def test_backward_full_size(name):
    """The 720p workloads (B=1, H=16, S=3600, D=128, bf16; T = 21 or 121) on the
    tensor-core path, in the launch configuration bench.py --bwd times, sampled
    slabs."""
    cfg = synth.CONFIGS[name]
    arr = synth.make_inputs(cfg)
    dO, dS = upstream(2024, cfg.B, cfg.H, cfg.T, cfg.S, cfg.D, True)
    check_case(arr, dO, dS, True, U.TOL_BF16, b_slabs=[(0, 0), (0, cfg.H - 1)])


def test_backward_bad_arguments_fail_loudly():
    arr = U.random_case(9, 1, 1, 2, 8, 16, bf16=False)
    d = U.dev_inputs(arr, False)
    with pytest.raises(api.GdnError):
        api.frame_scan_bwd(d["q"], d["k"], d["v"], d["beta"], d["gamma"], None, d["q"],
                           workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))


@pytest.mark.parametrize("fwd_kw", [dict(), dict(chunked=True), dict(sequential=True, overlap=False),
                                    dict(reverse=True, block_reset=True)])
def test_backward_from_saved_forward(fwd_kw):
    """The backward fed the forward call's workspace (no recompute) equals the
    recomputing backward and the oracle."""
    B, H, T, S, D = 1, 3, 9, 200, 128
    arr = U.random_case(61, B, H, T, S, D, bf16=True, state=True)
    dO, dS = upstream(62, B, H, T, S, D, True)
    d = U.dev_inputs(arr, True)
    d_out, d_s = U.to_dev(dO, True), torch.from_numpy(dS).cuda()
    ws = torch.empty(api.workspace_bytes(B, H, T, S, D, api.scan_flags(bf16=True, bidir=False)) +
                     (1 << 20), dtype=torch.uint8, device="cuda")
    api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"],
                          workspace=ws, save_for_backward=True, **fwd_kw)
    rkw = dict(reverse=fwd_kw.get("reverse", False), block_reset=fwd_kw.get("block_reset", False))
    got = api.frame_scan_bwd(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"], d_out,
                             d_s, saved_workspace=ws, **rkw)
    ref = api.frame_scan_bwd(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"], d_out,
                             d_s, **rkw)
    torch.cuda.synchronize()
    for name, g, r in zip(NAMES, got, ref):
        assert rel(U.host(g), U.host(r)) < 2e-3, name
    block = 3 if rkw["block_reset"] else 0
    for h in range(H):
        oref = O.frame_scan_bwd(U.widen(arr["q"][0, h], True), U.widen(arr["k"][0, h], True),
                                U.widen(arr["v"][0, h], True), arr["beta"][0, h].astype(np.float64),
                                arr["gamma"][0, h].astype(np.float64), arr["state"][0, h],
                                U.widen(dO[0, h], True), dS[0, h], reverse=rkw["reverse"],
                                block=block)
        for name, g, r in zip(NAMES, got, oref):
            assert rel(U.host(g[0, h]), r) < U.TOL_BF16, name
