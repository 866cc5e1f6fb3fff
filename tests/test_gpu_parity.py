"""GPU parity of the CUDA path against the float64 oracle, through the C ABI.

Small cases compare every output element; the full-size workloads (the 720p
configurations) run in the same launch configuration as bench.py and compare
sampled (b, h) slabs, which the oracle recomputes one by one.
"""

import numpy as np
import pytest
import torch

from frame_wise_gated_b200 import api, synth
from oracle import gdn_oracle as O
from tests import gdn_testutil as U

pytestmark = pytest.mark.gpu

PATHS = ["default", "simt"]


def tol(bf16):
    return U.TOL_BF16 if bf16 else U.TOL_FP32


def run_scan(d, path, **kw):
    return api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"],
                                 force_simt=(path == "simt"), **kw)


# ---------------------------------------------------------------------------
# step a2: per-frame contraction
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("D,S", [(16, 16), (32, 77), (64, 300), (128, 300), (128, 3600), (256, 200)])
def test_contract_stage(D, S, bf16, path):
    arr = U.random_case(100 + D + S, 1, 1, 5, S, D, bf16=bf16)
    k = U.to_dev(arr["k"][0, 0], bf16)
    v = U.to_dev(arr["v"][0, 0], bf16)
    beta = torch.from_numpy(arr["beta"][0, 0]).cuda()
    A, Uo = api.frame_contract(k, v, beta, force_simt=(path == "simt"))
    torch.cuda.synchronize()
    kk, vv = U.widen(arr["k"][0, 0], bf16), U.widen(arr["v"][0, 0], bf16)
    c = O.key_scale(D, S)
    bound = 1e-5 if (path == "simt" or not bf16) else 4e-3
    for t in range(5):
        Ar, Ur = O.frame_terms(c * kk[t], vv[t], arr["beta"][0, 0, t].astype(np.float64))
        assert U.rel_frob_per_frame(U.host(A[t])[None], Ar[None]) < bound
        assert U.rel_frob_per_frame(U.host(Uo[t])[None], Ur[None]) < bound


# ---------------------------------------------------------------------------
# step a3: span composites C = g (I - E), H
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("D,L", [(16, 3), (64, 8), (128, 8), (256, 5)])
def test_composites_stage(D, L, path):
    rng = np.random.default_rng(7 + D)
    N, S = 3, 40
    k = rng.standard_normal((N * L, S, D))
    v = rng.standard_normal((N * L, S, D))
    beta = rng.random((N * L, S))
    gamma = 0.9 + 0.1 * rng.random(N * L)
    c = O.key_scale(D, S)
    AU = [O.frame_terms(c * k[i], v[i], beta[i]) for i in range(N * L)]
    A = torch.tensor(np.stack([a for a, _ in AU]), dtype=torch.float32).cuda()
    Ut = torch.tensor(np.stack([u for _, u in AU]), dtype=torch.float32).cuda()
    gam = torch.tensor(gamma, dtype=torch.float32).cuda()
    E, Hc, g = api.chunk_composites(A, Ut, gam, L, force_simt=(path == "simt"))
    torch.cuda.synchronize()
    A64 = A.double().cpu().numpy()
    U64 = Ut.double().cpu().numpy()
    g64 = gam.double().cpu().numpy()
    for n in range(N):
        sl = slice(n * L, (n + 1) * L)
        # oracle composites from the same (fp32) A, U: C = prod gamma (I - A), H = scan from 0
        C = np.eye(D)
        Hm = np.zeros((D, D))
        for j in range(n * L, (n + 1) * L):
            M = g64[j] * (np.eye(D) - A64[j])
            C, Hm = C @ M, Hm @ M + U64[j]
        gg = float(g[n])
        assert gg == pytest.approx(np.prod(g64[sl]), rel=1e-6)
        Cg = gg * (np.eye(D) - U.host(E[n]))
        bound = 1e-5 if path == "simt" else 2e-3
        assert np.linalg.norm(Cg - C) / np.linalg.norm(C) < bound
        assert np.linalg.norm(U.host(Hc[n]) - Hm) / np.linalg.norm(Hm) < bound


# ---------------------------------------------------------------------------
# the whole scan on small cases, every mode
# ---------------------------------------------------------------------------

# Plans: "auto" lets the library choose (the sequential chains alongside the
# contraction on the tensor-core path at D = 128, else spans); the others force
# one plan. overlap=False keeps the sequential chains in their own launch.
MODES = {
    "auto": dict(),
    "chunked": dict(chunked=True),
    "chunk3": dict(chunk=3, chunked=True),
    "sequential": dict(sequential=True),
    "sequential_separate": dict(sequential=True, overlap=False),
    "reverse": dict(reverse=True),
    "reverse_chunked": dict(reverse=True, chunked=True),
    "reverse_block": dict(reverse=True, block_reset=True),
    "reverse_block_blocks": dict(reverse=True, block_reset=True, overlap=False),
    "forward_block": dict(block_reset=True, block=4),
    "forward_block_separate": dict(block_reset=True, block=4, sequential=True, overlap=False),
    "reverse_block_seq": dict(reverse=True, block_reset=True, sequential=True, overlap=False),
    "fused_replay": dict(fused_replay=True),
    "fused_replay_rev_block": dict(fused_replay=True, reverse=True, block_reset=True),
}


def oracle_kw(mode):
    kw = MODES[mode]
    return dict(reverse=kw.get("reverse", False),
                block=kw.get("block", 3) if kw.get("block_reset") else 0)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("D,bf16", [(16, False), (64, False), (128, False), (64, True),
                                    (128, True), (256, True)])
def test_scan_small(D, bf16, mode, path):
    B, H, T, S = 2, 1, 11, 200
    arr = U.random_case(1000 + D, B, H, T, S, D, bf16=bf16, state=True)
    d = U.dev_inputs(arr, bf16)
    out, st = run_scan(d, path, **MODES[mode])
    torch.cuda.synchronize()
    api.check_device_status()
    for b in range(B):
        o_ref, s_ref = U.oracle_slab(arr, b, 0, bf16, **oracle_kw(mode))
        assert U.rel_frob_per_frame(U.host(out[b, 0]), o_ref) < tol(bf16)
        assert U.rel_frob_per_frame(U.host(st[b, 0])[None], s_ref[None]) < tol(bf16)


def test_tiny_fp32_config_all_modes():
    cfg = synth.CONFIGS["tiny_fp32"]
    arr = synth.make_inputs(cfg)
    d = U.dev_inputs(arr, False)
    for mode in MODES:
        for chunk in (2, 3, 8):
            kw = dict(MODES[mode])
            kw.setdefault("chunk", chunk)
            out, st = run_scan(d, "default", **kw)
            o_ref, s_ref = U.oracle_slab(arr, 0, 0, False, **oracle_kw(mode))
            assert U.rel_frob_per_frame(U.host(out[0, 0]), o_ref) < U.TOL_FP32, (mode, chunk)
            assert U.rel_frob_per_frame(U.host(st[0, 0])[None], s_ref[None]) < U.TOL_FP32


def test_plain_entry_allocates_its_own_scratch():
    arr = U.random_case(5, 1, 2, 6, 64, 64, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    out, st = api.frame_scan_fwd(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"])
    out2, st2 = run_scan(d, "default")
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(st, st2)


def test_chunk_causal_streaming_blocks():
    """The chunk-causal inference step: one 3-frame block per call, the forward
    state carried from call to call (state_in = previous state_out), the
    reverse scan starting from zeros in every call (GDN_REV_STATE_IN with no
    reverse state). Three calls equal one bidirectional call over 9 frames
    (reset every 3 in reverse), and the oracle."""
    gh, gw, T = 6, 5, 9
    arr = U.random_case(71, 1, 2, T, gh * gw, 128, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    pro = dict(w_q=d["w_q"], w_k=d["w_k"], grid_h=gh, grid_w=gw)
    o_f, s_f, o_r, _ = run_scan(d, "default", prologue=pro, bidir=True, block_reset=True, block=3,
                                state_in_rev=None)
    st = d["state"]
    parts_f, parts_r = [], []
    for b0 in range(0, T, 3):
        sl = {n: d[n][:, :, b0:b0 + 3].contiguous() for n in ("q", "k", "v", "beta", "gamma")}
        of, st, orr, _ = api.frame_scan_fwd_ex(sl["q"], sl["k"], sl["v"], sl["beta"], sl["gamma"],
                                               st, prologue=pro, bidir=True, block_reset=True,
                                               block=3, state_in_rev=None)
        parts_f.append(of)
        parts_r.append(orr)
    torch.cuda.synchronize()
    gf, gr = torch.cat(parts_f, dim=2), torch.cat(parts_r, dim=2)
    assert U.rel_frob_per_frame(U.host(gf), U.host(o_f)) < 1e-3
    assert U.rel_frob_per_frame(U.host(gr), U.host(o_r)) < 1e-3
    assert U.rel_frob_per_frame(U.host(st)[None], U.host(s_f)[None]) < 1e-4
    for h in range(2):
        ref_f, ref_s = U.oracle_slab(arr, 0, h, True, prologue=(gw, 1e-6, 1e4))
        a0 = dict(arr, state=None)
        ref_r, _ = U.oracle_slab(a0, 0, h, True, prologue=(gw, 1e-6, 1e4), reverse=True, block=3)
        assert U.rel_frob_per_frame(U.host(gf[0, h]), ref_f) < U.TOL_BF16
        assert U.rel_frob_per_frame(U.host(gr[0, h]), ref_r) < U.TOL_BF16
        assert U.rel_frob_per_frame(U.host(st[0, h])[None], ref_s[None]) < U.TOL_BF16


def test_host_streaming_call():
    """frame_scan_fwd_host (host tensors, heads in chunks through ping-pong
    device buffers on three streams) equals the device call head by head, and
    the oracle."""
    arr = U.random_case(11, 2, 3, 5, 100, 128, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    ref_o, ref_s = run_scan(d, "default")
    torch.cuda.synchronize()
    h = {n: (t.cpu().pin_memory() if t is not None else None) for n, t in d.items()
         if n in ("q", "k", "v", "beta", "gamma", "state")}
    for hpc in (0, 1, 2, 4):  # 0: the library's default chunk
        o, s = api.frame_scan_fwd_host(h["q"], h["k"], h["v"], h["beta"], h["gamma"], h["state"],
                                       heads_per_chunk=hpc)
        assert not o.is_cuda and not s.is_cuda
        assert torch.equal(o, ref_o.cpu()) and torch.equal(s, ref_s.cpu()), hpc
    # pageable host memory (copies serialised) and no start state
    pg = {n: t.clone() for n, t in h.items() if t is not None}
    o2, s2 = api.frame_scan_fwd_host(pg["q"], pg["k"], pg["v"], pg["beta"], pg["gamma"], None,
                                     heads_per_chunk=2)
    ref2_o, ref2_s = api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"], None)
    torch.cuda.synchronize()
    assert torch.equal(o2, ref2_o.cpu()) and torch.equal(s2, ref2_s.cpu())
    for b in range(2):
        for hh in range(3):
            o_ref, s_ref = U.oracle_slab(arr, b, hh, True)
            assert U.rel_frob_per_frame(U.host(o[b, hh]), o_ref) < U.TOL_BF16


def test_streaming_split_equals_one_call():
    """A rollout split into two calls, carrying the state, equals one call."""
    arr = U.random_case(6, 1, 2, 12, 100, 64, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    out, st = run_scan(d, "default")
    part = lambda x, sl: x[:, :, sl].contiguous()
    a = {n: part(d[n], slice(0, 5)) for n in ("q", "k", "v", "beta", "gamma")}
    b = {n: part(d[n], slice(5, 12)) for n in ("q", "k", "v", "beta", "gamma")}
    o1, s1 = api.frame_scan_fwd_ex(a["q"], a["k"], a["v"], a["beta"], a["gamma"], d["state"])
    o2, s2 = api.frame_scan_fwd_ex(b["q"], b["k"], b["v"], b["beta"], b["gamma"], s1)
    torch.cuda.synchronize()
    ref = U.host(out)
    got = np.concatenate([U.host(o1), U.host(o2)], axis=2)
    assert U.rel_frob_per_frame(got, ref) < 1e-3
    assert U.rel_frob_per_frame(U.host(s2), U.host(st)) < 1e-4


def test_edge_sizes():
    for (T, S, D) in [(1, 1, 16), (1, 5, 64), (2, 129, 128), (9, 1, 128)]:
        arr = U.random_case(T * S + D, 1, 1, T, S, D, bf16=True, state=True)
        d = U.dev_inputs(arr, True)
        out, st = run_scan(d, "default")
        torch.cuda.synchronize()
        o_ref, s_ref = U.oracle_slab(arr, 0, 0, True)
        assert U.rel_frob_per_frame(U.host(out[0, 0]), o_ref) < U.TOL_BF16, (T, S, D)
        assert U.rel_frob_per_frame(U.host(st[0, 0])[None], s_ref[None]) < U.TOL_BF16


def test_bad_arguments_fail_loudly():
    arr = U.random_case(9, 1, 1, 2, 8, 16, bf16=False)
    d = U.dev_inputs(arr, False)
    with pytest.raises(api.GdnError):
        api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"], None,
                              out=d["q"])
    with pytest.raises(api.GdnError):
        api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"],
                              workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))


# ---------------------------------------------------------------------------
# prologue (a1), standalone and fused, and the bidirectional chunk-causal form (a7)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("D", [16, 64, 128, 256])
def test_prologue_stage(D, bf16):
    gh, gw = 5, 7
    arr = U.random_case(20 + D, 1, 2, 3, gh * gw, D, bf16=bf16)
    d = U.dev_inputs(arr, bf16)
    qh, kh = api.qk_prologue(d["q"], d["k"], d["w_q"], d["w_k"], gh, gw)
    torch.cuda.synchronize()
    q_ref, k_ref = O.qk_prologue(U.widen(arr["q"], bf16), U.widen(arr["k"], bf16),
                                 arr["w_q"], arr["w_k"], gw)
    bound = 1e-2 if bf16 else 1e-5
    assert U.rel_frob_per_frame(U.host(qh), q_ref) < bound
    assert U.rel_frob_per_frame(U.host(kh), k_ref) < bound


@pytest.mark.parametrize("overlap", [True, False])
@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("D", [64, 128])
def test_fused_prologue_bidirectional(D, path, overlap):
    gh, gw, T = 6, 5, 8
    arr = U.random_case(30 + D, 1, 2, T, gh * gw, D, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    pro = dict(w_q=d["w_q"], w_k=d["w_k"], grid_h=gh, grid_w=gw)
    out, st, out_r, st_r = run_scan(d, path, prologue=pro, bidir=True, block_reset=True, block=3,
                                    overlap=overlap)
    torch.cuda.synchronize()
    for h in range(2):
        o_f, s_f = U.oracle_slab(arr, 0, h, True, prologue=(gw, 1e-6, 1e4))
        o_r, s_r = U.oracle_slab(arr, 0, h, True, prologue=(gw, 1e-6, 1e4), reverse=True, block=3)
        assert U.rel_frob_per_frame(U.host(out[0, h]), o_f) < U.TOL_BF16
        assert U.rel_frob_per_frame(U.host(out_r[0, h]), o_r) < U.TOL_BF16
        assert U.rel_frob_per_frame(U.host(st[0, h])[None], s_f[None]) < U.TOL_BF16
        assert U.rel_frob_per_frame(U.host(st_r[0, h])[None], s_r[None]) < U.TOL_BF16


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("path", PATHS)
def test_fused_prologue_one_direction(path, reverse):
    """Fused prologue with a single scan direction, on a 9 x 23 grid: 207
    tokens span several contraction stages and readout tiles with a ragged
    tail, and rows of the grid straddle tile boundaries."""
    gh, gw, T = 9, 23, 5
    arr = U.random_case(41, 1, 2, T, gh * gw, 128, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    pro = dict(w_q=d["w_q"], w_k=d["w_k"], grid_h=gh, grid_w=gw)
    block = 2 if reverse else 3
    out, st = run_scan(d, path, prologue=pro, reverse=reverse, block_reset=reverse, block=block)
    torch.cuda.synchronize()
    for h in range(2):
        o_ref, s_ref = U.oracle_slab(arr, 0, h, True, prologue=(gw, 1e-6, 1e4), reverse=reverse,
                                     block=block if reverse else 0)
        assert U.rel_frob_per_frame(U.host(out[0, h]), o_ref) < U.TOL_BF16
        assert U.rel_frob_per_frame(U.host(st[0, h])[None], s_ref[None]) < U.TOL_BF16


@pytest.mark.parametrize("overlap", [True, False])
def test_fused_prologue_bidirectional_multitile(overlap):
    """Bidirectional form on a 9 x 23 grid (several tiles, ragged tail)."""
    gh, gw, T = 9, 23, 7
    arr = U.random_case(43, 1, 2, T, gh * gw, 128, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    pro = dict(w_q=d["w_q"], w_k=d["w_k"], grid_h=gh, grid_w=gw)
    out, st, out_r, st_r = run_scan(d, "default", prologue=pro, bidir=True, block_reset=True,
                                    block=3, overlap=overlap)
    torch.cuda.synchronize()
    for h in range(2):
        o_f, s_f = U.oracle_slab(arr, 0, h, True, prologue=(gw, 1e-6, 1e4))
        o_r, s_r = U.oracle_slab(arr, 0, h, True, prologue=(gw, 1e-6, 1e4), reverse=True, block=3)
        assert U.rel_frob_per_frame(U.host(out[0, h]), o_f) < U.TOL_BF16
        assert U.rel_frob_per_frame(U.host(out_r[0, h]), o_r) < U.TOL_BF16
        assert U.rel_frob_per_frame(U.host(st[0, h])[None], s_f[None]) < U.TOL_BF16
        assert U.rel_frob_per_frame(U.host(st_r[0, h])[None], s_r[None]) < U.TOL_BF16


@pytest.mark.parametrize("bidir_prologue", [False, True])
def test_readout_three_part_units(bidir_prologue):
    """Frames of 1496 tokens (a 34 x 44 grid: 12 readout tiles, the last one
    88 tokens): each frame-head's tiles go to three work units of 4 tiles, so
    unit boundaries, ragged tails and several units per CTA all occur; forward
    scan, or the fused-prologue bidirectional form."""
    gh, gw, T = 34, 44, 4
    arr = U.random_case(47, 1, 3, T, gh * gw, 128, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    if bidir_prologue:
        pro = dict(w_q=d["w_q"], w_k=d["w_k"], grid_h=gh, grid_w=gw)
        out, st, out_r, st_r = run_scan(d, "default", prologue=pro, bidir=True, block_reset=True,
                                        block=3)
    else:
        out, st = run_scan(d, "default")
    torch.cuda.synchronize()
    for h in range(3):
        if bidir_prologue:
            o_ref, s_ref = U.oracle_slab(arr, 0, h, True, prologue=(gw, 1e-6, 1e4))
            o_rr, _ = U.oracle_slab(arr, 0, h, True, prologue=(gw, 1e-6, 1e4), reverse=True, block=3)
            assert U.rel_frob_per_frame(U.host(out_r[0, h]), o_rr) < U.TOL_BF16
        else:
            o_ref, s_ref = U.oracle_slab(arr, 0, h, True)
        assert U.rel_frob_per_frame(U.host(out[0, h]), o_ref) < U.TOL_BF16
        assert U.rel_frob_per_frame(U.host(st[0, h])[None], s_ref[None]) < U.TOL_BF16


# ---------------------------------------------------------------------------
# full-size workloads, as bench.py launches them; sampled slabs vs the oracle
# ---------------------------------------------------------------------------

FULL = [
    ("clip5s_720p", {}),
    ("clip5s_720p", {"chunked": True}),
    ("clip5s_720p", {"fused_replay": True}),
    ("rollout60s_720p", {}),
    ("rollout60s_720p", {"chunked": True}),
    ("rollout60s_720p", {"sequential": True, "overlap": False}),
    ("prologue_bidir_720p", {}),
    ("prologue_bidir_720p", {"overlap": False}),
    ("prologue_ucpe_bidir_720p", {}),
    ("sweep_d64", {}),
    ("sweep_d256", {}),
    ("sweep_d256", {"chunked": True}),
    ("stream_block3_720p", {}),
    ("stream_block3_720p", {"overlap": False}),
]


@pytest.mark.parametrize("name,kw", FULL, ids=[n + "".join("-" + k for k in kw) for n, kw in FULL])
def test_full_size_sampled(name, kw):
    cfg = synth.CONFIGS[name]
    arr = synth.make_inputs(cfg)
    d = U.dev_inputs(arr, cfg.bf16)
    cam = None
    if cfg.ucpe:  # camera matrices of the synthetic trajectory (queries D^T, keys D^-1)
        cam = synth.make_camera(cfg.B, cfg.T, cfg.grid_h, cfg.grid_w, cfg.seed)
    if cfg.prologue:
        pro = dict(w_q=d["w_q"], w_k=d["w_k"], grid_h=cfg.grid_h, grid_w=cfg.grid_w)
        if cam is not None:
            pro["ucpe_q"], pro["ucpe_k"] = (torch.from_numpy(m).cuda() for m in cam)
        out, st, out_r, st_r = run_scan(d, "default", prologue=pro, bidir=True,
                                        block_reset=True, block=cfg.bidir_block, **kw)
    else:
        out, st = run_scan(d, "default", **kw)
    torch.cuda.synchronize()
    api.check_device_status()
    assert torch.isfinite(out.float()).all()
    rng = np.random.default_rng(sum(name.encode()))
    samples = {(0, 0), (cfg.B - 1, cfg.H - 1)}
    samples.add((int(rng.integers(cfg.B)), int(rng.integers(cfg.H))))
    for (b, h) in sorted(samples):
        if cfg.prologue:
            pro_o = (cfg.grid_w, 1e-6, 1e4)
            o_ref, s_ref = U.oracle_slab(arr, b, h, True, prologue=pro_o, ucpe=cam)
            o_rr, s_rr = U.oracle_slab(arr, b, h, True, prologue=pro_o, reverse=True,
                                       block=cfg.bidir_block, ucpe=cam)
            assert U.rel_frob_per_frame(U.host(out_r[b, h]), o_rr) < U.TOL_BF16
            assert U.rel_frob_per_frame(U.host(st_r[b, h])[None], s_rr[None]) < U.TOL_BF16
        else:
            o_ref, s_ref = U.oracle_slab(arr, b, h, cfg.bf16)
        assert U.rel_frob_per_frame(U.host(out[b, h]), o_ref) < tol(cfg.bf16), (b, h)
        assert U.rel_frob_per_frame(U.host(st[b, h])[None], s_ref[None]) < tol(cfg.bf16)


def test_chunked_matches_sequential_full_size():
    cfg = synth.CONFIGS["rollout60s_720p"]
    arr = synth.make_inputs(cfg)
    d = U.dev_inputs(arr, True)
    o1, s1 = run_scan(d, "default", chunked=True)
    for kw in (dict(sequential=True), dict(sequential=True, overlap=False)):
        o2, s2 = run_scan(d, "default", **kw)
        torch.cuda.synchronize()
        num = (o1.float() - o2.float()).flatten(3).norm(dim=-1)
        den = o2.float().flatten(3).norm(dim=-1)
        assert float((num / den).max()) < 5e-3, kw
        assert float(((s1 - s2).flatten(2).norm(dim=-1) / s2.flatten(2).norm(dim=-1)).max()) < 1e-3


def _phase_launches(fn):
    api.profile_enable(True)
    fn()
    torch.cuda.synchronize()
    rec = api.profile_read()
    api.profile_enable(False)
    return {k: v[1] for k, v in rec.items()}


def test_plan_selection():
    """The library runs the chains alongside the contraction exactly where the
    plan says so, and its result equals the separate-launch sequential scan."""
    arr = U.random_case(77, 1, 3, 9, 150, 128, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    got = {}
    for name, kw in (("auto", {}), ("chunked", dict(chunked=True)),
                     ("separate", dict(sequential=True, overlap=False))):
        def call(kw=kw, name=name):
            got[name] = run_scan(d, "default", **kw)
        n = _phase_launches(call)
        assert n["contract_scan"] == (1 if name == "auto" else 0), (name, n)
        assert n["contract"] == (0 if name == "auto" else 1), (name, n)
    o_a, s_a = got["auto"]
    o_s, s_s = got["separate"]
    assert U.rel_frob_per_frame(U.host(o_a), U.host(o_s)) < 1e-3
    assert U.rel_frob_per_frame(U.host(s_a)[None], U.host(s_s)[None]) < 1e-4
    # more chains than a quarter of the SMs: the chunked plan
    many = U.random_case(78, 1, 40, 10, 64, 128, bf16=True)
    dm = U.dev_inputs(many, True)
    n = _phase_launches(lambda: run_scan(dm, "default"))
    assert n["contract_scan"] == 0 and n["compose"] == 1, n


def test_plan_selection_d256():
    """D = 256: whole-scan tensor-core chains by default (one launch, no span
    composition); spans when asked for; both equal the oracle."""
    arr = U.random_case(79, 2, 1, 10, 90, 256, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    for kw, expect_compose in (({}, 0), (dict(chunked=True), 1)):
        res = {}
        n = _phase_launches(lambda: res.setdefault("r", run_scan(d, "default", **kw)))
        assert n["compose"] == expect_compose and n["scan"] == 1, (kw, n)
        out, st = res["r"]
        for b in range(2):
            o_ref, s_ref = U.oracle_slab(arr, b, 0, True)
            assert U.rel_frob_per_frame(U.host(out[b, 0]), o_ref) < U.TOL_BF16, kw
            assert U.rel_frob_per_frame(U.host(st[b, 0])[None], s_ref[None]) < U.TOL_BF16, kw


@pytest.mark.parametrize("H,T,S", [(3, 7, 1000), (1, 5, 300), (2, 3, 600), (4, 9, 2000)])
def test_token_split_ranges_repeated_calls(H, T, S):
    """Token-split plan (at most a quarter of the SMs in frame-heads): sizes
    whose parts do not divide a frame's stages evenly, three calls in a row
    (a stale accumulator would show up from the second call on)."""
    arr = U.random_case(300 + H * T, 1, H, T, S, 128, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    refs = [U.oracle_slab(arr, 0, h, True) for h in range(H)]
    for call in range(3):
        out, st = api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"])
        torch.cuda.synchronize()
        api.check_device_status()
        for h, (o_ref, s_ref) in enumerate(refs):
            assert U.rel_frob_per_frame(U.host(out[0, h]), o_ref) < U.TOL_BF16, (call, h)
            assert U.rel_frob_per_frame(U.host(st[0, h])[None], s_ref[None]) < U.TOL_BF16, (call, h)
