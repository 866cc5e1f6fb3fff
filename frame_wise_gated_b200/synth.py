"""Seeded synthetic inputs for the frame scan, shared by the tests, the bench
and the oracle checks.

This module draws random numbers and rounds them to bf16; it holds none of
the scan's arithmetic. Every (b, h) slab has its own PCG64 stream seeded by
(seed, b, h), so any slab can be regenerated alone: the oracle recomputes
sampled slabs of a full-size workload without drawing the rest.

Shapes follow the pages' 720p workload: an 80 x 45 latent grid (S = 3600
tokens per frame, "Jiayun's Blog" section 2.1), T = 21 / 61 / 121 latent frames,
and a reset block of 3 frames (chunk_size: 3, "SANA-WM 世界模型实战指南"
section 七). They stand in for GDN-layer activations of that model, whose
weights and data are not available.
"""

from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os

import numpy as np

__all__ = ["Config", "CONFIGS", "bf16_round_bits", "bf16_bits_to_f32",
           "make_slab", "make_inputs", "make_state", "make_weights", "make_camera"]


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    B: int
    H: int
    T: int
    S: int
    D: int
    grid_h: int
    grid_w: int
    bf16: bool
    seed: int
    beta_dist: str = "uniform"      # "uniform" U[0,1] or "beta22" Beta(2,2)
    gamma_lo: float = 0.9           # gamma ~ U[gamma_lo, 1]
    state_sigma: float = 0.0        # S_0 ~ N(0, sigma^2) per entry, 0 -> zeros
    prologue: bool = False          # raw q, k go through the fused prologue
    bidir_block: int = 0            # >0: forward scan + reverse scan reset every block
    ucpe: bool = False              # the prologue includes the camera encoding

    @property
    def frame_heads(self) -> int:
        return self.B * self.H * self.T

    @property
    def tokens(self) -> int:
        return self.B * self.H * self.T * self.S


CONFIGS = {
    "tiny_fp32": Config("tiny_fp32", 1, 1, 8, 16, 16, 4, 4, False, 1),
    "clip5s_720p": Config("clip5s_720p", 1, 16, 21, 3600, 128, 45, 80, True, 2),
    "rollout60s_720p": Config("rollout60s_720p", 1, 16, 121, 3600, 128, 45, 80, True, 3),
    "prologue_bidir_720p": Config("prologue_bidir_720p", 1, 16, 121, 3600, 128, 45, 80, True, 4,
                                  prologue=True, bidir_block=3),
    # config 4 plus the camera encoding (per-token ray-local transforms of a
    # synthetic camera trajectory, see make_camera)
    "prologue_ucpe_bidir_720p": Config("prologue_ucpe_bidir_720p", 1, 16, 121, 3600, 128, 45, 80,
                                       True, 9, prologue=True, bidir_block=3, ucpe=True),
    "prologue_bidir_clip5s_720p": Config("prologue_bidir_clip5s_720p", 1, 16, 21, 3600, 128, 45,
                                         80, True, 7, prologue=True, bidir_block=3),
    # one call of the chunk-causal streaming step: one 3-frame block, forward
    # state carried in, reverse scan inside the block
    "stream_block3_720p": Config("stream_block3_720p", 1, 16, 3, 3600, 128, 45, 80, True, 8,
                                 prologue=True, bidir_block=3, state_sigma=0.1),
    "sweep_d64": Config("sweep_d64", 4, 32, 61, 3600, 64, 45, 80, True, 5,
                        beta_dist="beta22", gamma_lo=0.8, state_sigma=0.1),
    "sweep_d256": Config("sweep_d256", 4, 8, 61, 3600, 256, 45, 80, True, 6,
                         beta_dist="beta22", gamma_lo=0.8, state_sigma=0.1),
}


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact widening)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def make_slab(cfg: Config, b: int, h: int):
    """Draws one (b, h) slab: q, k, v [T, S, D] float32 ~ N(0, 1) (raw q, k
    for the prologue configs), beta [T, S], gamma [T]. Draw order: q, k, v,
    beta, gamma. q, k, v are returned as bf16 bits (uint16) for bf16 configs,
    float32 otherwise."""
    rng = np.random.default_rng([cfg.seed, b, h])
    shape = (cfg.T, cfg.S, cfg.D)
    out = {}
    for name in ("q", "k", "v"):
        x = rng.standard_normal(shape, dtype=np.float32)
        out[name] = bf16_round_bits(x) if cfg.bf16 else x
    if cfg.beta_dist == "beta22":
        out["beta"] = rng.beta(2.0, 2.0, size=(cfg.T, cfg.S)).astype(np.float32)
    else:
        out["beta"] = rng.random((cfg.T, cfg.S), dtype=np.float32)
    out["gamma"] = (cfg.gamma_lo + (1.0 - cfg.gamma_lo) *
                    rng.random(cfg.T, dtype=np.float32)).astype(np.float32)
    return out


def make_state(cfg: Config):
    """Initial state S_0 [B, H, D, D] float32, or None when it is zero."""
    if cfg.state_sigma == 0.0:
        return None
    rng = np.random.default_rng([cfg.seed, 1_000_003])
    return (cfg.state_sigma * rng.standard_normal((cfg.B, cfg.H, cfg.D, cfg.D))).astype(np.float32)


def make_weights(cfg: Config):
    """RMSNorm weights (w_q, w_k) [D] float32 ~ U[0.5, 1.5]."""
    rng = np.random.default_rng([cfg.seed, 1_000_004])
    return ((0.5 + rng.random(cfg.D)).astype(np.float32),
            (0.5 + rng.random(cfg.D)).astype(np.float32))


def make_inputs(cfg: Config, threads: int | None = None):
    """All slabs stacked: q, k, v [B, H, T, S, D] (bf16 bits or float32),
    beta [B, H, T, S], gamma [B, H, T], plus state (or None) and weights."""
    B, H, T, S, D = cfg.B, cfg.H, cfg.T, cfg.S, cfg.D
    et = np.uint16 if cfg.bf16 else np.float32
    arr = {n: np.empty((B, H, T, S, D), et) for n in ("q", "k", "v")}
    arr["beta"] = np.empty((B, H, T, S), np.float32)
    arr["gamma"] = np.empty((B, H, T), np.float32)

    def fill(bh):
        b, h = divmod(bh, H)
        sl = make_slab(cfg, b, h)
        for n, x in sl.items():
            arr[n][b, h] = x

    n = threads or min(16, os.cpu_count() or 1)
    with _cf.ThreadPoolExecutor(max_workers=n) as ex:
        list(ex.map(fill, range(B * H)))
    arr["state"] = make_state(cfg)
    arr["w_q"], arr["w_k"] = make_weights(cfg)
    return arr


def _rot(axis: int, a: float) -> np.ndarray:
    c, s_ = np.cos(a), np.sin(a)
    i, j = [(1, 2), (0, 2), (0, 1)][axis]
    R = np.eye(3)
    R[i, i] = R[j, j] = c
    R[i, j], R[j, i] = -s_, s_
    return R


def make_camera(B: int, T: int, grid_h: int, grid_w: int, seed: int):
    """Synthetic camera geometry for the camera encoding: per batch b a smooth
    trajectory over the T latent frames (yaw and pitch growing with t, the
    centre on a small arc, |c| <= 0.5) seen through a pinhole camera with a
    90-degree horizontal field of view on the grid_h x grid_w latent grid.
    For token s = y * grid_w + x of frame t the ray through the pixel centre
    defines a ray-local frame (z along the ray, x perpendicular to it and to
    the camera's up axis); D_{t,s} maps world coordinates into that frame.
    Returns (M_q, M_k) [B, T, S, 4, 4] float32: D^T for queries and D^-1 for
    keys. Geometry only: the transforms are inputs of the prologue."""
    rng = np.random.default_rng([seed, 1_000_005])
    S = grid_h * grid_w
    f = grid_w / 2.0
    ys, xs = np.divmod(np.arange(S), grid_w)
    d = np.stack([(xs + 0.5 - grid_w / 2.0) / f, (ys + 0.5 - grid_h / 2.0) / f, np.ones(S)], -1)
    d /= np.linalg.norm(d, axis=-1, keepdims=True)
    up = np.array([0.0, 1.0, 0.0])
    xr = np.cross(up, d)
    xr /= np.linalg.norm(xr, axis=-1, keepdims=True)
    yr = np.cross(d, xr)
    R_ray = np.stack([xr, yr, d], 1)                     # [S, 3, 3]: camera -> ray-local
    Mq = np.empty((B, T, S, 4, 4), np.float32)
    Mk = np.empty((B, T, S, 4, 4), np.float32)
    for b in range(B):
        yaw0, pitch0 = rng.uniform(-0.5, 0.5, 2)
        for t in range(T):
            R_t = _rot(1, yaw0 + 0.03 * t) @ _rot(0, pitch0 + 0.01 * t)   # camera -> world
            c = 0.4 * np.array([np.sin(0.05 * t), 0.1 * np.sin(0.1 * t), 1.0 - np.cos(0.05 * t)])
            Rw = R_ray @ R_t.T                                           # world -> ray-local
            Dm = np.zeros((S, 4, 4))
            Dm[:, :3, :3] = Rw
            Dm[:, :3, 3] = -Rw @ c
            Dm[:, 3, 3] = 1.0
            Di = np.zeros((S, 4, 4))
            Di[:, :3, :3] = np.transpose(Rw, (0, 2, 1))
            Di[:, :3, 3] = c
            Di[:, 3, 3] = 1.0
            Mq[b, t] = np.transpose(Dm, (0, 2, 1))
            Mk[b, t] = Di
    return Mq, Mk
