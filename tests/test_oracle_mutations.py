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
