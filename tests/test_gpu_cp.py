"""Context parallelism on the GPU kernels: R ranks' shards computed on one
GPU (the all-gather replaced by stacking), through gdn_cp_shard_composite and
gdn_cp_prefix, equal one scan over the whole sequence and the oracle."""

import numpy as np
import pytest
import torch

from frame_wise_gated_b200 import api
from tests import gdn_testutil as U

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D,bf16,R", [(64, True, 2), (128, True, 3), (128, False, 2),
                                      (256, True, 2), (32, False, 4)])
def test_cp_shards_equal_one_scan(D, bf16, R):
    B, H, T, S = 1, 2, 12, 150
    arr = U.random_case(90 + D + R, B, H, T, S, D, bf16=bf16, state=True)
    d = U.dev_inputs(arr, bf16)
    full_o, full_s = api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"],
                                           d["state"])
    per = T // R
    parts = [{n: d[n][:, :, r * per:(r + 1) * per].contiguous()
              for n in ("q", "k", "v", "beta", "gamma")} for r in range(R)]
    maps = [api.cp_shard_composite(p["k"], p["v"], p["beta"], p["gamma"]) for p in parts]
    E_all = torch.stack([m[0] for m in maps])
    H_all = torch.stack([m[1] for m in maps])
    g_all = torch.stack([m[2] for m in maps])
    outs, st = [], None
    for r, p in enumerate(parts):
        s0 = api.cp_prefix(E_all, H_all, g_all, d["state"], r)
        o, st = api.frame_scan_fwd_ex(p["q"], p["k"], p["v"], p["beta"], p["gamma"], s0)
        outs.append(o)
    torch.cuda.synchronize()
    got = torch.cat(outs, dim=2)
    tol = U.TOL_BF16 if bf16 else U.TOL_FP32
    assert U.rel_frob_per_frame(U.host(got), U.host(full_o)) < tol
    assert U.rel_frob_per_frame(U.host(st)[None], U.host(full_s)[None]) < tol
    for h in range(H):
        o_ref, s_ref = U.oracle_slab(arr, 0, h, bf16)
        assert U.rel_frob_per_frame(U.host(got[0, h]), o_ref) < tol
        assert U.rel_frob_per_frame(U.host(st[0, h])[None], s_ref[None]) < tol


@pytest.mark.parametrize("R,rev", [(2, "default"), (4, "zeros")])
def test_cp_bidirectional_shards_equal_one_call(R, rev):
    """The bidirectional chunk-causal form (reverse reset every 3 frames) over
    R shards of whole blocks (12 frames: shards of 6 or 3), each shard's forward started from the prefix of
    the earlier shards' maps and its reverse local (seeded on the last shard
    only), equals one bidirectional call over the whole sequence and the
    oracle -- what frame_scan_bidir_cp computes on R ranks."""
    B, H, T, S, D = 1, 2, 12, 150, 128
    arr = U.random_case(95 + R, B, H, T, S, D, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    kw = dict(bidir=True, block_reset=True, block=3)
    rev_kw = {} if rev == "default" else dict(state_in_rev=None)
    full = api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"],
                                 **kw, **rev_kw)
    per = T // R
    parts = [{n: d[n][:, :, r * per:(r + 1) * per].contiguous()
              for n in ("q", "k", "v", "beta", "gamma")} for r in range(R)]
    maps = [api.cp_shard_composite(p["k"], p["v"], p["beta"], p["gamma"]) for p in parts]
    E_all, H_all, g_all = (torch.stack([m[i] for m in maps]) for i in range(3))
    res = []
    for r, p in enumerate(parts):
        s0 = api.cp_prefix(E_all, H_all, g_all, d["state"], r)
        seed = (d["state"] if rev == "default" else None) if r == R - 1 else None
        res.append(api.frame_scan_fwd_ex(p["q"], p["k"], p["v"], p["beta"], p["gamma"], s0,
                                         state_in_rev=seed, **kw))
    torch.cuda.synchronize()
    got_f = torch.cat([x[0] for x in res], dim=2)
    got_r = torch.cat([x[2] for x in res], dim=2)
    assert U.rel_frob_per_frame(U.host(got_f), U.host(full[0])) < U.TOL_BF16
    assert U.rel_frob_per_frame(U.host(got_r), U.host(full[2])) < U.TOL_BF16
    assert U.rel_frob_per_frame(U.host(res[-1][1])[None], U.host(full[1])[None]) < U.TOL_BF16
    assert U.rel_frob_per_frame(U.host(res[0][3])[None], U.host(full[3])[None]) < U.TOL_BF16
    a0 = arr if rev == "default" else dict(arr, state=None)
    for h in range(H):
        o_ref, _ = U.oracle_slab(arr, 0, h, True)
        o_rr, _ = U.oracle_slab(a0, 0, h, True, reverse=True, block=3)
        assert U.rel_frob_per_frame(U.host(got_f[0, h]), o_ref) < U.TOL_BF16
        assert U.rel_frob_per_frame(U.host(got_r[0, h]), o_rr) < U.TOL_BF16
