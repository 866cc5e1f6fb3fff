"""The shared input generator: bf16 rounding and per-slab determinism (CPU)."""

import numpy as np
import torch

from frame_wise_gated_b200 import synth


def test_bf16_rounding_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -1 - 2 ** -8, 0.0, -0.0], np.float32)])
    bits = synth.bf16_round_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, ref)
    back = synth.bf16_bits_to_f32(bits)
    np.testing.assert_array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_slabs_are_independent_and_repeatable():
    cfg = synth.CONFIGS["tiny_fp32"]
    a = synth.make_slab(cfg, 0, 0)
    b = synth.make_slab(cfg, 0, 0)
    for n in a:
        np.testing.assert_array_equal(a[n], b[n])
    full = synth.make_inputs(cfg)
    np.testing.assert_array_equal(full["q"][0, 0], a["q"])
    assert full["state"] is None


def test_distributions():
    cfg = synth.Config("t", 1, 2, 4, 500, 16, 20, 25, True, 9, beta_dist="beta22",
                       gamma_lo=0.8, state_sigma=0.1)
    x = synth.make_inputs(cfg)
    assert x["q"].dtype == np.uint16
    assert 0.0 <= x["beta"].min() and x["beta"].max() <= 1.0
    assert abs(x["beta"].mean() - 0.5) < 0.02
    assert 0.8 <= x["gamma"].min() and x["gamma"].max() <= 1.0
    assert abs(x["state"].std() - 0.1) < 0.01
    q = synth.bf16_bits_to_f32(x["q"])
    assert abs(q.std() - 1.0) < 0.02
    assert 0.5 <= x["w_q"].min() and x["w_q"].max() <= 1.5
