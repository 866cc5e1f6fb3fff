"""Canary guard regions: no kernel writes outside the buffers it is given.

compute-sanitizer is closed on this machine, so out-of-bounds writes are looked
for this way instead: every output (out, out_rev, the states, the gradients)
and the caller's workspace is a view into the middle of a larger buffer whose
64 KiB before and after hold a byte pattern; after each plan runs, the
pattern must be intact. Sizes leave a ragged last token tile. Each guarded
result must also equal the same call on plain buffers (bit for bit, all these
plans being deterministic), so the guarded run did its work.
"""

import math

import pytest
import torch

from frame_wise_gated_b200 import api, synth
from tests import gdn_testutil as U

pytestmark = pytest.mark.gpu

G = 1 << 16
PAT = 0xA5


class Guarded:
    def __init__(self, shape, dtype):
        el = torch.empty((), dtype=dtype).element_size()
        self.n = math.prod(shape) * el
        self.raw = torch.full((G + self.n + G,), PAT, dtype=torch.uint8, device="cuda")
        self.view = self.raw[G:G + self.n].view(dtype).view(shape)

    def intact(self):
        return bool((self.raw[:G] == PAT).all()) and bool((self.raw[G + self.n:] == PAT).all())


def guarded_ws(need):
    return Guarded((max(need, 256),), torch.uint8)


# At D = 128 with at most 37 frame-heads (a quarter of 148 SMs) and 193 or
# more tokens per frame the library cuts each frame-head's tokens over several
# CTAs (the token-split plan); every case but "token_split" stays above that.
FWD = [
    # name, B, H, T, S, D, bf16, keywords
    ("overlap", 1, 4, 12, 1000, 128, True, dict()),
    ("overlap_rev_block", 1, 4, 10, 1000, 128, True, dict(reverse=True, block_reset=True)),
    ("chunked", 1, 3, 17, 700, 128, True, dict(chunked=True)),
    ("sequential_no_overlap", 1, 3, 14, 700, 128, True, dict(sequential=True, overlap=False)),
    ("token_split", 1, 2, 3, 600, 128, True, dict()),
    ("fused_replay", 1, 2, 16, 700, 128, True, dict(chunked=True, fused_replay=True)),
    ("d64_chunked", 2, 3, 9, 700, 64, True, dict()),
    ("d256_sequential", 1, 2, 5, 700, 256, True, dict()),
    ("simt_fp32_d32", 1, 2, 5, 300, 32, False, dict()),
]


@pytest.mark.parametrize("case", FWD, ids=[c[0] for c in FWD])
def test_forward_writes_stay_inside_buffers(case):
    name, B, H, T, S, D, bf16, kw = case
    arr = U.random_case(100 + FWD.index(case), B, H, T, S, D, bf16=bf16, state=True)
    d = U.dev_inputs(arr, bf16)
    dt = torch.bfloat16 if bf16 else torch.float32
    out = Guarded((B, H, T, S, D), dt)
    st = Guarded((B, H, D, D), torch.float32)
    flags = api.scan_flags(bf16=bf16, **kw)
    ws = guarded_ws(api.workspace_bytes(B, H, T, S, D, flags))
    api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"],
                          out=out.view, state_out=st.view, workspace=ws.view, **kw)
    ref_o, ref_s = api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"],
                                         d["state"], **kw)
    torch.cuda.synchronize()
    api.check_device_status()
    for g, what in ((out, "out"), (st, "state_out"), (ws, "workspace")):
        assert g.intact(), (name, what)
    if name == "token_split":  # partial sums meet in atomic adds: order varies
        assert U.rel_frob_per_frame(U.host(out.view).reshape(-1, S, D),
                                    U.host(ref_o).reshape(-1, S, D)) < U.TOL_BF16
    else:
        assert torch.equal(out.view, ref_o) and torch.equal(st.view, ref_s), name


@pytest.mark.parametrize("camera", [False, True])
@pytest.mark.parametrize("bidir", [True, False])
def test_fused_prologue_writes_stay_inside_buffers(bidir, camera):
    B, H, T, gh, gw, D = 1, 3, 13, 20, 50, 128
    S = gh * gw
    arr = U.random_case(61, B, H, T, S, D, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    pro = dict(w_q=d["w_q"], w_k=d["w_k"], grid_h=gh, grid_w=gw)
    if camera:
        mq, mk = synth.make_camera(B, T, gh, gw, 61)
        pro["ucpe_q"], pro["ucpe_k"] = torch.from_numpy(mq).cuda(), torch.from_numpy(mk).cuda()
    kw = dict(bidir=True, block_reset=True) if bidir else dict()
    out, out_r = Guarded((B, H, T, S, D), torch.bfloat16), Guarded((B, H, T, S, D), torch.bfloat16)
    st, st_r = Guarded((B, H, D, D), torch.float32), Guarded((B, H, D, D), torch.float32)
    flags = api.scan_flags(bf16=True, prologue=True, **kw) | (api.UCPE if camera else 0)
    ws = guarded_ws(api.workspace_bytes(B, H, T, S, D, flags))
    extra = dict(out_rev=out_r.view, state_out_rev=st_r.view) if bidir else {}
    got = api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"],
                                prologue=pro, out=out.view, state_out=st.view, workspace=ws.view,
                                **extra, **kw)
    ref = api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"],
                                prologue=pro, **kw)
    torch.cuda.synchronize()
    api.check_device_status()
    guards = [(out, "out"), (st, "state_out"), (ws, "workspace")]
    if bidir:
        guards += [(out_r, "out_rev"), (st_r, "state_out_rev")]
    for g, what in guards:
        assert g.intact(), what
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


@pytest.mark.parametrize("D", [128, 64])
def test_backward_writes_stay_inside_buffers(D):
    B, H, T, S = 1, 3, 13, 1000
    arr = U.random_case(62, B, H, T, S, D, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    g = torch.Generator(device="cuda").manual_seed(5)
    d_out = torch.randn((B, H, T, S, D), device="cuda", generator=g).to(torch.bfloat16)
    gr = {n: Guarded((B, H, T, S, D), torch.bfloat16) for n in ("dq", "dk", "dv")}
    gr["dbeta"] = Guarded((B, H, T, S), torch.float32)
    gr["dgamma"] = Guarded((B, H, T), torch.float32)
    gr["d_state_in"] = Guarded((B, H, D, D), torch.float32)
    flags = api.scan_flags(bf16=True, reverse=True, block_reset=True)
    need = int(api.lib().gdn_bwd_workspace_bytes(B, H, T, S, D, flags))
    ws = guarded_ws(need)
    got = api.frame_scan_bwd(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"], d_out,
                             reverse=True, block_reset=True, workspace=ws.view,
                             grads={n: x.view for n, x in gr.items()})
    ref = api.frame_scan_bwd(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"], d_out,
                             reverse=True, block_reset=True)
    torch.cuda.synchronize()
    api.check_device_status()
    for n, x in list(gr.items()) + [("workspace", ws)]:
        assert x.intact(), n
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
