"""GPU parity of the camera encoding (UCPE) composed with the 2-D RoPE, in the
standalone prologue and in the fused scan, against the float64 oracle
(its pins: tests/test_oracle_pins.py). Camera matrices come from the seeded
synthetic trajectory and pinhole rays of synth.make_camera.

Metric as everywhere: per frame ||x_gpu - x_ref||_F / ||x_ref||_F, bounds
1e-4 (fp32 inputs) and 1e-2 (bf16 inputs).
"""

import numpy as np
import pytest
import torch

from frame_wise_gated_b200 import api, synth
from oracle import gdn_oracle as O
from tests import gdn_testutil as U

pytestmark = pytest.mark.gpu


def camera(B, T, gh, gw, seed):
    Mq, Mk = synth.make_camera(B, T, gh, gw, seed)
    return (Mq, Mk), (torch.from_numpy(Mq).cuda(), torch.from_numpy(Mk).cuda())


@pytest.mark.parametrize("D", [16, 64, 128, 256])
@pytest.mark.parametrize("bf16", [True, False])
def test_prologue_ucpe_matches_oracle(D, bf16):
    B, H, T, gh, gw = 2, 2, 3, 9, 23
    S = gh * gw
    arr = U.random_case(90 + D, B, H, T, S, D, bf16=bf16)
    d = U.dev_inputs(arr, bf16)
    cam_h, cam_d = camera(B, T, gh, gw, 90 + D)
    qh, kh = api.qk_prologue(d["q"], d["k"], d["w_q"], d["w_k"], gh, gw, ucpe=cam_d)
    torch.cuda.synchronize()
    tol = U.TOL_BF16 if bf16 else U.TOL_FP32
    for b in range(B):
        for h in range(H):
            rq, rk = O.qk_prologue(U.widen(arr["q"][b, h], bf16), U.widen(arr["k"][b, h], bf16),
                                   arr["w_q"], arr["w_k"], gw, ucpe=(cam_h[0][b], cam_h[1][b]))
            assert U.rel_frob_per_frame(U.host(qh[b, h]), rq) < tol
            assert U.rel_frob_per_frame(U.host(kh[b, h]), rk) < tol


@pytest.mark.parametrize("bidir", [True, False])
def test_fused_scan_with_ucpe_matches_oracle(bidir):
    B, H, T, gh, gw, D = 1, 3, 7, 20, 50, 128
    S = gh * gw
    arr = U.random_case(95, B, H, T, S, D, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    cam_h, cam_d = camera(B, T, gh, gw, 95)
    pro = dict(w_q=d["w_q"], w_k=d["w_k"], grid_h=gh, grid_w=gw, ucpe_q=cam_d[0], ucpe_k=cam_d[1])
    kw = dict(bidir=True, block_reset=True) if bidir else dict()
    res = api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"],
                                prologue=pro, **kw)
    torch.cuda.synchronize()
    api.check_device_status()
    for h in range(H):
        o_ref, s_ref = U.oracle_slab(arr, 0, h, True, prologue=(gw, 1e-6, 1e4), ucpe=cam_h)
        assert U.rel_frob_per_frame(U.host(res[0][0, h]), o_ref) < U.TOL_BF16
        assert U.rel_frob_per_frame(U.host(res[1][0, h])[None], s_ref[None]) < U.TOL_BF16
        if bidir:
            r_ref, sr_ref = U.oracle_slab(arr, 0, h, True, reverse=True, block=3,
                                          prologue=(gw, 1e-6, 1e4), ucpe=cam_h)
            assert U.rel_frob_per_frame(U.host(res[2][0, h]), r_ref) < U.TOL_BF16
            assert U.rel_frob_per_frame(U.host(res[3][0, h])[None], sr_ref[None]) < U.TOL_BF16


def test_ucpe_with_identity_equals_rope_on_the_upper_half():
    """Identity camera matrices: channels [0, D/2) are only normalised, and
    [D/2, D) carry the RoPE of D/2 channels (same kernel, no tolerance beyond
    the bf16 output rounding of identical values)."""
    B, H, T, gh, gw, D = 1, 2, 2, 9, 23, 128
    S = gh * gw
    arr = U.random_case(97, B, H, T, S, D, bf16=True)
    d = U.dev_inputs(arr, True)
    eye = torch.eye(4, device="cuda").expand(B, T, S, 4, 4).contiguous()
    qh, kh = api.qk_prologue(d["q"], d["k"], d["w_q"], d["w_k"], gh, gw, ucpe=(eye, eye))
    torch.cuda.synchronize()
    for b_h in range(H):
        rq, rk = O.qk_prologue(U.widen(arr["q"][0, b_h], True), U.widen(arr["k"][0, b_h], True),
                               arr["w_q"], arr["w_k"], gw,
                               ucpe=(np.tile(np.eye(4), (T, S, 1, 1)),) * 2)
        assert U.rel_frob_per_frame(U.host(qh[0, b_h]), rq) < U.TOL_BF16


def test_ucpe_argument_errors():
    arr = U.random_case(98, 1, 1, 2, 16, 16, bf16=True)
    d = U.dev_inputs(arr, True)
    pro = dict(w_q=d["w_q"], w_k=d["w_k"], grid_h=4, grid_w=4,
               ucpe_q=torch.zeros((1, 2, 16, 4, 4), device="cuda"),
               ucpe_k=torch.zeros((1, 2, 16, 4, 3), device="cuda"))
    with pytest.raises(ValueError):
        api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"], prologue=pro)


@pytest.mark.parametrize("ucpe", [False, True])
@pytest.mark.parametrize("plan", ["auto", "chunked", "separate"])
def test_standalone_prologue_then_scan_with_scaled_keys(plan, ucpe):
    """The two-call form: gdn_qk_prologue(_ucpe) writes q^, k^ (k^ carrying the
    key scale), then the scan runs with GDN_KEYS_SCALED in each plan."""
    B, H, T, gh, gw, D = 1, 3, 7, 20, 50, 128
    S = gh * gw
    arr = U.random_case(96, B, H, T, S, D, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    cam_h, cam_d = camera(B, T, gh, gw, 96)
    qh, kh = api.qk_prologue(d["q"], d["k"], d["w_q"], d["w_k"], gh, gw,
                             ucpe=cam_d if ucpe else None)
    kw = {"auto": {}, "chunked": dict(chunked=True),
          "separate": dict(sequential=True, overlap=False)}[plan]
    out, st = api.frame_scan_fwd_ex(qh, kh, d["v"], d["beta"], d["gamma"], d["state"],
                                    keys_scaled=True, **kw)
    torch.cuda.synchronize()
    api.check_device_status()
    for h in range(H):
        o_ref, s_ref = U.oracle_slab(arr, 0, h, True, prologue=(gw, 1e-6, 1e4),
                                     ucpe=cam_h if ucpe else None)
        assert U.rel_frob_per_frame(U.host(out[0, h]), o_ref) < U.TOL_BF16, h
        assert U.rel_frob_per_frame(U.host(st[0, h])[None], s_ref[None]) < U.TOL_BF16, h
