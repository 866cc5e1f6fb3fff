"""Helpers shared by the GPU parity tests: moving seeded inputs to the device,
running the oracle on chosen (b, h) slabs, and the error metric.

Error metric (spec tolerance): max over (b, h, t) of
||O_gpu - O_ref||_F / ||O_ref||_F, and max over (b, h) of the same for the
final state; bounds 1e-4 for fp32 inputs, 1e-2 for bf16 inputs.
"""

from __future__ import annotations

import numpy as np
import torch

from frame_wise_gated_b200 import synth
from oracle import gdn_oracle as O

TOL_FP32 = 1e-4
TOL_BF16 = 1e-2


def widen(x: np.ndarray, bf16: bool) -> np.ndarray:
    """Input array as the exact float64 values the device sees."""
    return synth.bf16_bits_to_f32(x).astype(np.float64) if bf16 else np.asarray(x, np.float64)


def to_dev(x: np.ndarray, bf16: bool) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    if bf16 and x.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.cuda()


def dev_inputs(arr: dict, bf16: bool):
    d = {n: to_dev(arr[n], bf16) for n in ("q", "k", "v")}
    d["beta"] = torch.from_numpy(arr["beta"]).cuda()
    d["gamma"] = torch.from_numpy(arr["gamma"]).cuda()
    d["state"] = None if arr.get("state") is None else torch.from_numpy(arr["state"]).cuda()
    if "w_q" in arr:
        d["w_q"] = torch.from_numpy(arr["w_q"]).cuda()
        d["w_k"] = torch.from_numpy(arr["w_k"]).cuda()
    return d


def rel_frob_per_frame(got: np.ndarray, ref: np.ndarray) -> float:
    """max over leading frames of ||got - ref||_F / ||ref||_F; arrays [..., S, D]."""
    got = np.asarray(got, np.float64).reshape(-1, got.shape[-2] * got.shape[-1])
    ref = np.asarray(ref, np.float64).reshape(-1, ref.shape[-2] * ref.shape[-1])
    num = np.linalg.norm(got - ref, axis=1)
    den = np.linalg.norm(ref, axis=1)
    return float(np.max(num / np.maximum(den, 1e-300)))


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.cpu().numpy().astype(np.float64)


def random_case(seed, B, H, T, S, D, *, bf16, state=False, beta_hi=1.0, gamma_lo=0.9):
    """Seeded small case in the configs' distributions (q, k, v ~ N(0,1),
    beta ~ U[0, beta_hi], gamma ~ U[gamma_lo, 1]); bf16 inputs as RNE bits."""
    rng = np.random.default_rng(seed)
    arr = {}
    for n in ("q", "k", "v"):
        x = rng.standard_normal((B, H, T, S, D), dtype=np.float32)
        arr[n] = synth.bf16_round_bits(x) if bf16 else x
    arr["beta"] = (beta_hi * rng.random((B, H, T, S), dtype=np.float32)).astype(np.float32)
    arr["gamma"] = (gamma_lo + (1 - gamma_lo) * rng.random((B, H, T), dtype=np.float32)).astype(np.float32)
    arr["state"] = (0.1 * rng.standard_normal((B, H, D, D))).astype(np.float32) if state else None
    arr["w_q"] = (0.5 + rng.random(D)).astype(np.float32)
    arr["w_k"] = (0.5 + rng.random(D)).astype(np.float32)
    return arr


def oracle_slab(arr, b, h, bf16, *, reverse=False, block=0, keys_scaled=False, prologue=None,
                ucpe=None):
    """Oracle output and final state for slab (b, h). prologue = (grid_w, eps, base);
    ucpe = (M_q, M_k) [B, T, S, 4, 4] camera matrices (with the prologue)."""
    q = widen(arr["q"][b, h], bf16)
    k = widen(arr["k"][b, h], bf16)
    v = widen(arr["v"][b, h], bf16)
    if prologue is not None:
        grid_w, eps, base = prologue
        cam = None if ucpe is None else (ucpe[0][b], ucpe[1][b])
        q, k = O.qk_prologue(q, k, arr["w_q"], arr["w_k"], grid_w, eps=eps, base=base, ucpe=cam)
        keys_scaled = True
    s0 = None if arr.get("state") is None else arr["state"][b, h]
    return O.frame_scan(q, k, v, arr["beta"][b, h].astype(np.float64),
                        arr["gamma"][b, h].astype(np.float64), s0, reverse=reverse,
                        block=block, keys_scaled=keys_scaled)
