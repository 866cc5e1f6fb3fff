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
