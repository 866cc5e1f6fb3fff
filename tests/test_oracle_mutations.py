"""Plants plausible mistakes in copies of the oracle's scan and checks that
the pins catch every one of them (CPU only; the oracle itself is untouched)."""

import json
import os

import numpy as np
import pytest

from oracle import gdn_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def make_scan(mutation):
    def scan(q, k, v, beta, gamma, state_in=None, *, keys_scaled=False):
        q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
        T, S, D = q.shape
        c = 1.0 if keys_scaled else O.key_scale(D, S)
        if mutation == "scale_sqrt_S_only":
            c = 1.0 / np.sqrt(S)
        St = np.zeros((D, D)) if state_in is None else np.array(state_in, np.float64)
        out = np.empty((T, S, D))
        for t in range(T):
            kh = c * k[t]
            bk = beta[t][:, None] * kh
            A = kh.T @ bk
            U = v[t].T @ bk
            if mutation == "U_transposed":
                U = U.T
            if mutation == "beta_dropped_in_U":
                U = v[t].T @ kh
            if mutation == "left_multiply":
                St = gamma[t] * (St - A @ St) + U
            elif mutation == "plus_sign":
                St = gamma[t] * (St + St @ A) + U
            elif mutation == "gamma_on_U":
                St = gamma[t] * (St - St @ A + U)
            elif mutation == "gamma_dropped":
                St = St - St @ A + U
            else:
                St = gamma[t] * (St - St @ A) + U
            if mutation == "readout_untransposed":
                out[t] = q[t] @ St
            elif mutation == "readout_pre_update":
                out[t] = q[t] @ (St - U).T
            else:
                out[t] = q[t] @ St.T
        return out, St
    return scan


def pins_pass(scan):
    ok = True
    for name in ("delta_rule_2x2.json", "scalar_geometric.json"):
        g = json.load(open(os.path.join(GOLD, name)))
        o, st = scan(np.array(g["q"]), np.array(g["k"]), np.array(g["v"]),
                     np.array(g["beta"]), np.array(g["gamma"]))
        ok &= np.allclose(o, g["expected_out"], atol=1e-9) and np.allclose(st, g["expected_state"], atol=1e-9)
    rng = np.random.default_rng(5)
    T, D = 9, 6
    q, k, v = (rng.standard_normal((T, 1, D)) for _ in range(3))
    beta, gamma = rng.random((T, 1)), 0.9 + 0.1 * rng.random(T)
    s0 = rng.standard_normal((D, D))
    o, st = scan(q, k, v, beta, gamma, s0)
    o2, st2 = O.token_wise_gdn(q[:, 0], k[:, 0] / np.sqrt(D), v[:, 0], beta[:, 0], gamma, s0)
    ok &= np.allclose(o[:, 0], o2, atol=1e-9) and np.allclose(st, st2, atol=1e-9)
    D, S = 8, 3
    basis, _ = np.linalg.qr(rng.standard_normal((D, D)))
    kh = basis[:S]
    vv = rng.standard_normal((S, D))
    o, st = scan(kh[None], np.sqrt(D * S) * kh[None], vv[None], np.ones((1, S)), np.ones(1),
                 rng.standard_normal((D, D)))
    ok &= np.allclose(o[0], vv, atol=1e-9)
    return bool(ok)


def test_unmutated_copy_passes():
    assert pins_pass(make_scan(None))


@pytest.mark.parametrize("mutation", [
    "U_transposed", "beta_dropped_in_U", "left_multiply", "plus_sign", "gamma_on_U",
    "gamma_dropped", "readout_untransposed", "readout_pre_update", "scale_sqrt_S_only"])
def test_pins_catch_mutation(mutation):
    assert not pins_pass(make_scan(mutation))


# --- the prologue: planted mistakes in copies of rmsnorm / rope2d ----------

def make_rmsnorm(mutation):
    def rmsnorm(x, w, eps=1e-6):
        x = np.asarray(x, np.float64)
        w = np.asarray(w, np.float64)
        ms = np.mean(x * x, axis=-1, keepdims=True)
        if mutation == "eps_outside_root":
            return x / (np.sqrt(ms) + eps) * w
        if mutation == "eps_dropped":
            return x / np.sqrt(ms) * w
        if mutation == "weight_before_norm":
            xw = x * w
            return xw / np.sqrt(np.mean(xw * xw, axis=-1, keepdims=True) + eps)
        return x / np.sqrt(ms + eps) * w
    return rmsnorm


def make_rope2d(mutation):
    def rope2d(x, grid_w, base=10000.0):
        x = np.array(x, np.float64)
        S, D = x.shape[-2], x.shape[-1]
        half = D // 2
        s = np.arange(S)
        pos_y, pos_x = s // grid_w, s % grid_w
        if mutation == "axes_swapped":
            pos_y, pos_x = pos_x, pos_y
        out = x.copy()
        for i in range(D // 4):
            expo = 2.0 * i / (D if mutation == "full_D_exponent" else half)
            theta = base ** (-expo)
            for off, pos in ((0, pos_y), (half, pos_x)):
                phi = pos * theta
                cs, sn = np.cos(phi), np.sin(phi)
                if mutation == "sign_flipped":
                    sn = -sn
                if mutation == "rotate_half_pairs":   # pairs (i, i + D/4) instead of (2i, 2i+1)
                    ia, ib = off + i, off + i + D // 4
                else:
                    ia, ib = off + 2 * i, off + 2 * i + 1
                a, b = x[..., ia], x[..., ib]
                out[..., ia] = a * cs - b * sn
                out[..., ib] = a * sn + b * cs
        return out
    return rope2d


def prologue_pins_pass(rmsnorm, rope2d):
    ok = True
    g = json.load(open(os.path.join(GOLD, "rope2d_pair1.json")))
    for c in g["cases"]:
        x = np.zeros((c["S"], g["D"]))
        x[g["token"]] = g["x_in"]
        ok &= np.allclose(rope2d(x, c["grid_w"], g["base"])[g["token"]], c["expected"], atol=1e-12)
    g = json.load(open(os.path.join(GOLD, "rmsnorm_eps.json")))
    ok &= np.allclose(rmsnorm(np.array(g["x"]), np.array(g["w"]), eps=g["eps"]), g["expected"],
                      atol=1e-14)
    # the first pair of each half turns by exactly pos radians
    x = np.zeros((8, 8))
    x[:, 0] = 1.0
    x[:, 4] = 1.0
    y = rope2d(x, 4)
    ok &= np.allclose(y[6, :2], [np.cos(1.0), np.sin(1.0)]) and np.allclose(
        y[6, 4:6], [np.cos(2.0), np.sin(2.0)])
    return bool(ok)


def test_unmutated_prologue_copy_passes():
    assert prologue_pins_pass(make_rmsnorm(None), make_rope2d(None))
    # and the copies agree with the oracle itself
    rng = np.random.default_rng(11)
    x, w = rng.standard_normal((12, 16)), 0.5 + rng.random(16)
    np.testing.assert_allclose(make_rmsnorm(None)(x, w, 0.3), O.rmsnorm(x, w, 0.3), rtol=1e-15)
    np.testing.assert_allclose(make_rope2d(None)(x, 4), O.rope2d(x, 4), rtol=1e-15)


@pytest.mark.parametrize("mutation", ["eps_outside_root", "eps_dropped", "weight_before_norm"])
def test_pins_catch_rmsnorm_mutation(mutation):
    assert not prologue_pins_pass(make_rmsnorm(mutation), make_rope2d(None))


@pytest.mark.parametrize("mutation", ["full_D_exponent", "axes_swapped", "sign_flipped",
                                      "rotate_half_pairs"])
def test_pins_catch_rope_mutation(mutation):
    assert not prologue_pins_pass(make_rmsnorm(None), make_rope2d(mutation))


# --- the camera encoding: planted mistakes in copies of ucpe_rope ------------

def make_ucpe(mutation):
    def ucpe_rope(x, M, grid_w, base=10000.0):
        x = np.array(x, np.float64)
        M = np.asarray(M, np.float64)
        if mutation == "transposed":
            M = np.swapaxes(M, -1, -2)
        D = x.shape[-1]
        h = D // 2
        lo, hi = (slice(h, D), slice(0, h)) if mutation == "halves_swapped" else (slice(0, h), slice(h, D))
        out = x.copy()
        xs = x[..., lo]
        ys = out[..., lo]
        for b in range(h // 4):
            if mutation == "strided_blocks":   # block b = channels b, b + D/8, ... instead of 4b..4b+3
                idx = [b + j * (h // 4) for j in range(4)]
            else:
                idx = list(range(4 * b, 4 * b + 4))
            ys[..., idx] = np.einsum("...ij,...j->...i", M, xs[..., idx])
        out[..., lo] = ys
        out[..., hi] = O.rope2d(x[..., hi], grid_w, base)
        return out
    return ucpe_rope


def ucpe_pins_pass(fn):
    g = json.load(open(os.path.join(GOLD, "ucpe_rope_d8.json")))
    x = np.zeros((g["S"], g["D"]))
    x[g["token"]] = g["x_in"]
    M = np.tile(np.eye(4), (g["S"], 1, 1))
    M[g["token"]] = g["M"]
    ok = np.allclose(fn(x, M, g["grid_w"], g["base"])[g["token"]], g["expected"], atol=1e-12)
    rng = np.random.default_rng(43)
    x = rng.standard_normal((6, 32))
    y = fn(x, np.tile(np.eye(4), (6, 1, 1)), 3)
    ok &= np.array_equal(y[:, :16], x[:, :16]) and np.allclose(y[:, 16:], O.rope2d(x[:, 16:], 3))
    # index loops at D = 16: two camera blocks of 4 consecutive channels
    x, M = rng.standard_normal((6, 16)), rng.standard_normal((6, 4, 4))
    y = fn(x, M, 3)
    for s_ in range(6):
        for b in range(2):
            for i in range(4):
                ok &= abs(y[s_][4 * b + i] - sum(M[s_][i][j] * x[s_][4 * b + j] for j in range(4))) < 1e-12
    return bool(ok)


def test_unmutated_ucpe_copy_passes():
    assert ucpe_pins_pass(make_ucpe(None))
    rng = np.random.default_rng(44)
    x, M = rng.standard_normal((6, 32)), rng.standard_normal((6, 4, 4))
    np.testing.assert_allclose(make_ucpe(None)(x, M, 3), O.ucpe_rope(x, M, 3), rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("mutation", ["transposed", "halves_swapped", "strided_blocks"])
def test_pins_catch_ucpe_mutation(mutation):
    assert not ucpe_pins_pass(make_ucpe(mutation))
