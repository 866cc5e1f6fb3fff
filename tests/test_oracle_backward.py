"""Pins of the oracle's backward (frame_scan_bwd): the pages print no
gradient, so the adjoint is checked against central finite differences of the
pinned forward scan, for every input, in every scan mode; and plausible
mistakes planted in a copy of the adjoint are shown to fail that check.
CPU only."""

import numpy as np
import pytest

from oracle import gdn_oracle as O


def _case(seed, T=4, S=3, D=3, state=True):
    rng = np.random.default_rng(seed)
    x = dict(q=rng.standard_normal((T, S, D)), k=rng.standard_normal((T, S, D)),
             v=rng.standard_normal((T, S, D)), beta=rng.random((T, S)),
             gamma=0.8 + 0.2 * rng.random(T),
             s0=0.3 * rng.standard_normal((D, D)) if state else None)
    dO = rng.standard_normal((T, S, D))
    dS = rng.standard_normal((D, D))
    return x, dO, dS


def _loss(x, dO, dS, **kw):
    o, st = O.frame_scan(x["q"], x["k"], x["v"], x["beta"], x["gamma"], x["s0"], **kw)
    return float(np.sum(o * dO) + (np.sum(st * dS) if dS is not None else 0.0))


def _fd(x, dO, dS, name, h=1e-6, **kw):
    g = np.zeros_like(x[name])
    it = np.nditer(x[name], flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        xp = {n: (None if a is None else np.array(a)) for n, a in x.items()}
        xm = {n: (None if a is None else np.array(a)) for n, a in x.items()}
        xp[name][i] += h
        xm[name][i] -= h
        g[i] = (_loss(xp, dO, dS, **kw) - _loss(xm, dO, dS, **kw)) / (2 * h)
    return g


NAMES = ("q", "k", "v", "beta", "gamma", "s0")


def _check(bwd, x, dO, dS, tol=1e-6, **kw):
    got = bwd(x["q"], x["k"], x["v"], x["beta"], x["gamma"], x["s0"], dO, dS, **kw)
    worst = 0.0
    for name, g in zip(NAMES, got):
        if x[name] is None:
            continue
        ref = _fd(x, dO, dS, name, **kw)
        err = np.max(np.abs(g - ref)) / max(1e-12, np.max(np.abs(ref)))
        worst = max(worst, err)
    return worst


MODES = [dict(), dict(reverse=True), dict(block=2), dict(reverse=True, block=3),
         dict(keys_scaled=True)]


@pytest.mark.parametrize("kw", MODES, ids=["forward", "reverse", "block2", "reverse_block3",
                                           "keys_scaled"])
@pytest.mark.parametrize("with_state", [True, False])
def test_backward_matches_finite_differences(kw, with_state):
    x, dO, dS = _case(3, state=with_state)
    assert _check(O.frame_scan_bwd, x, dO, dS, **kw) < 1e-6
    # the state gradient alone, and the output gradient alone
    assert _check(O.frame_scan_bwd, x, np.zeros_like(dO), dS, **kw) < 1e-6
    assert _check(O.frame_scan_bwd, x, dO, None, **kw) < 1e-6


def test_backward_single_token_frames():
    """S = 1: the frame-wise scan is token-wise GDN; its gradient must still
    match finite differences (a different regime: rank-one A_t)."""
    x, dO, dS = _case(8, T=6, S=1, D=4)
    assert _check(O.frame_scan_bwd, x, dO, dS) < 1e-6


def test_backward_zero_beta_is_pure_decay():
    """beta = 0: S_t = gamma_t S_{t-1}, so dq, dk, dv vanish only through A, U
    (dk = dv = 0) and dgamma_t = <dM_t, I> = tr(S_{t-1}^T G_t)."""
    x, dO, dS = _case(9)
    x["beta"] = np.zeros_like(x["beta"])
    dq, dk, dv, db, dg, ds0 = O.frame_scan_bwd(x["q"], x["k"], x["v"], x["beta"], x["gamma"],
                                               x["s0"], dO, dS)
    assert np.all(dk == 0) and np.all(dv == 0)
    assert _check(O.frame_scan_bwd, x, dO, dS) < 1e-6


def _mutant(mutation):
    """A copy of the adjoint (forward scan order only) with one planted mistake."""
    def bwd(q, k, v, beta, gamma, s0, d_out, d_state_out=None):
        T, S, D = q.shape
        c = O.key_scale(D, S)
        X = np.zeros((D, D)) if s0 is None else np.array(s0)
        prev, As = [], []
        for t in range(T):
            A, U = O.frame_terms(c * k[t], v[t], beta[t])
            prev.append(X)
            As.append(A)
            X = gamma[t] * (X - X @ A) + U
        states = prev[1:] + [X]
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        db, dg = np.zeros_like(beta), np.zeros_like(gamma)
        Gn, ds0, I = None, np.zeros((D, D)), np.eye(D)
        for t in range(T - 1, -1, -1):
            G = d_out[t].T @ q[t]
            if t == T - 1 and d_state_out is not None:
                G = G + d_state_out
            if Gn is not None:
                G = G + Gn
            dq[t] = d_out[t] @ (prev[t] if mutation == "dq_pre_update" else states[t])
            A = As[t]
            dM = prev[t].T @ G
            if mutation == "dM_untransposed":
                dM = prev[t] @ G
            dA = -gamma[t] * dM
            dg[t] = np.sum(dM * (I - A)) * (-1 if mutation == "dgamma_sign" else 1)
            kh = c * k[t]
            sym = dA if mutation == "dA_not_symmetrised" else dA + dA.T
            bcol = np.ones_like(beta[t])[:, None] if mutation == "beta_dropped_dv" else beta[t][:, None]
            dk[t] = c * beta[t][:, None] * (kh @ sym.T + v[t] @ G)
            dv[t] = bcol * (kh @ G.T)
            db[t] = np.einsum("sd,sd->s", kh, kh @ dA.T) + np.einsum("sd,sd->s", v[t] @ G, kh)
            gcar = 1.0 if mutation == "carry_without_gamma" else gamma[t]
            carry = G @ (gcar * (I - A)).T
            if t == 0:
                ds0 = carry
            else:
                Gn = carry
        return dq, dk, dv, db, dg, ds0
    return bwd


@pytest.mark.parametrize("mutation", ["none", "dq_pre_update", "dM_untransposed", "dgamma_sign",
                                      "dA_not_symmetrised", "beta_dropped_dv",
                                      "carry_without_gamma"])
def test_planted_backward_mistakes_are_caught(mutation):
    x, dO, dS = _case(21, T=4, S=3, D=3)
    err = _check(_mutant(mutation), x, dO, dS)
    if mutation == "none":
        assert err < 1e-6
    else:
        assert err > 1e-3, mutation
