"""Accuracy of the fused prologue's RoPE (cos, sin) pairs over the whole
position range, against float64 cos / sin of the exact angle
pos * base^(-2i/(D/2)) (reading R10 of the 2-D RoPE).

Both paths compute the angle in fp32, so their error grows with the angle:
the fp32 frequency (powf, a few ulp) and the fp32 product pos * theta each
add about 2^-24 of it. On top of that the table path's sine/cosine adds about
1e-7, and the range-reduced path (Cody-Waite reduction to [-pi, pi], then the
hardware sine/cosine) about 4e-7. Bound used: 4e-7 * angle + 1e-6.
"""

import ctypes

import numpy as np
import pytest
import torch

from frame_wise_gated_b200 import api

pytestmark = pytest.mark.gpu


def _eval(npos, D, base, reduced):
    cs = torch.empty((D // 4, npos, 2), device="cuda", dtype=torch.float32)
    rc = api.lib().gdn_rope_eval(npos, D, ctypes.c_float(base), int(reduced),
                                 ctypes.c_void_p(cs.data_ptr()), None)
    assert rc == 0, api.lib().gdn_last_error()
    torch.cuda.synchronize()
    return cs.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("reduced", [False, True])
def test_rope_cos_sin_error_bound(D, reduced):
    npos, base = 4096, 10000.0
    got = _eval(npos, D, base, reduced)
    i = np.arange(D // 4)[:, None]
    pos = np.arange(npos)[None, :]
    ang = pos * base ** (-2.0 * i / (D // 2))
    err = np.maximum(np.abs(got[..., 0] - np.cos(ang)), np.abs(got[..., 1] - np.sin(ang)))
    bound = 4e-7 * ang + 1e-6
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), (worst, err[worst], bound[worst])
    # on the 720p latent grid (positions below 80) the pairs are good to 5e-5
    assert err[:, :80].max() < 5e-5


def test_rope_eval_rejects_bad_arguments():
    L = api.lib()
    cs = torch.empty(64, device="cuda")
    assert L.gdn_rope_eval(0, 128, ctypes.c_float(1e4), 0, ctypes.c_void_p(cs.data_ptr()),
                           None) == api.GDN_ERR_INVALID
    assert L.gdn_rope_eval(4, 48, ctypes.c_float(1e4), 0, ctypes.c_void_p(cs.data_ptr()),
                           None) == api.GDN_ERR_INVALID
    assert L.gdn_rope_eval(4, 128, ctypes.c_float(1e4), 0, None, None) == api.GDN_ERR_INVALID
