"""Pins of the float64 oracle to facts outside itself (CPU only).

Each test ties the oracle to something the pages or the mathematics fix: a
hand-worked example, a published special case, a closed form, a theorem the
pages state, or an invariant. A plausible slip in the oracle (a dropped term,
a wrong sign, a transposed operand, a wrong index or scale) fails at least one.
"""

import json
import os

import numpy as np
import pytest

from oracle import gdn_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def rand_case(rng, T, S, D, beta_hi=1.0):
    q = rng.standard_normal((T, S, D))
    k = rng.standard_normal((T, S, D))
    v = rng.standard_normal((T, S, D))
    beta = beta_hi * rng.random((T, S))
    gamma = 0.9 + 0.1 * rng.random(T)
    return q, k, v, beta, gamma


# --- hand-worked golden fixtures -------------------------------------------

@pytest.mark.parametrize("name", ["delta_rule_2x2.json", "scalar_geometric.json"])
def test_golden_fixture(name):
    g = json.load(open(os.path.join(GOLD, name)))
    out, st = O.frame_scan(np.array(g["q"]), np.array(g["k"]), np.array(g["v"]),
                           np.array(g["beta"]), np.array(g["gamma"]))
    np.testing.assert_allclose(out, np.array(g["expected_out"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(st, np.array(g["expected_state"]), rtol=0, atol=1e-12)


# --- published special case: S = 1 is token-wise GDN ("Jiayun's Blog" 2.1) ---

def test_single_token_frames_reduce_to_token_wise_gdn():
    rng = np.random.default_rng(11)
    T, D = 17, 8
    q, k, v, beta, gamma = rand_case(rng, T, 1, D)
    s0 = rng.standard_normal((D, D))
    out, st = O.frame_scan(q, k, v, beta, gamma, s0)
    o_tok, st_tok = O.token_wise_gdn(q[:, 0], k[:, 0] / np.sqrt(D), v[:, 0],
                                     beta[:, 0], gamma, s0)
    np.testing.assert_allclose(out[:, 0], o_tok, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(st, st_tok, rtol=1e-12, atol=1e-12)


# --- delta rule: with orthonormal scaled keys and beta = gamma = 1 the state
#     maps each key exactly onto its value and leaves other directions alone --

def test_delta_rule_writes_values_at_keys():
    rng = np.random.default_rng(12)
    D, S = 8, 3
    basis, _ = np.linalg.qr(rng.standard_normal((D, D)))
    k_hat = basis[:S]                          # orthonormal rows
    k = np.sqrt(D * S) * k_hat                 # the oracle divides by sqrt(D*S)
    v = rng.standard_normal((S, D))
    s0 = rng.standard_normal((D, D))
    out, st = O.frame_scan(k_hat[None], k[None], v[None], np.ones((1, S)),
                           np.ones(1), s0)
    np.testing.assert_allclose(st @ k_hat.T, v.T, atol=1e-12)   # S k^_s = v_s
    np.testing.assert_allclose(out[0], v, atol=1e-12)           # query = key -> value
    x = basis[S:]                                               # orthogonal complement
    np.testing.assert_allclose(st @ x.T, s0 @ x.T, atol=1e-12)


# --- closed form: keys giving A = a I make the recurrence a geometric series --

def test_isotropic_keys_geometric_series():
    rng = np.random.default_rng(13)
    D = S = 4
    T = 20
    a, g = 0.3, 0.93
    k1 = np.sqrt(D * S) * np.sqrt(a) * np.eye(D)       # K^ = sqrt(a) I -> A = a I
    v1 = rng.standard_normal((S, D))
    U = v1.T @ (np.sqrt(a) * np.eye(D))               # V^T beta K^ with beta = 1
    s0 = rng.standard_normal((D, D))
    k = np.repeat(k1[None], T, 0)
    v = np.repeat(v1[None], T, 0)
    q = rng.standard_normal((T, S, D))
    out, st = O.frame_scan(q, k, v, np.ones((T, S)), np.full(T, g), s0)
    r = g * (1 - a)
    closed = r ** T * s0 + U * (1 - r ** T) / (1 - r)
    np.testing.assert_allclose(st, closed, rtol=1e-12, atol=1e-12)
    t = 6
    St = r ** (t + 1) * s0 + U * (1 - r ** (t + 1)) / (1 - r)
    np.testing.assert_allclose(out[t], q[t] @ St.T, rtol=1e-12, atol=1e-12)


def test_key_scale_closed_form():
    assert O.key_scale(16, 16) == pytest.approx(1 / 16, rel=1e-15)
    assert O.key_scale(128, 3600) == pytest.approx(1 / np.sqrt(460800), rel=1e-15)


# --- invariants --------------------------------------------------------------

def test_beta_zero_is_pure_decay():
    rng = np.random.default_rng(14)
    T, S, D = 6, 5, 4
    q, k, v, beta, gamma = rand_case(rng, T, S, D)
    s0 = rng.standard_normal((D, D))
    out, st = O.frame_scan(q, k, v, np.zeros((T, S)), gamma, s0)
    np.testing.assert_allclose(st, np.prod(gamma) * s0, rtol=1e-13)
    for t in range(T):
        np.testing.assert_allclose(out[t], q[t] @ (np.prod(gamma[:t + 1]) * s0).T, rtol=1e-12)


def test_gamma_one_beta_zero_keeps_state():
    rng = np.random.default_rng(15)
    T, S, D = 5, 3, 4
    q, k, v, _, _ = rand_case(rng, T, S, D)
    s0 = rng.standard_normal((D, D))
    _, st = O.frame_scan(q, k, v, np.zeros((T, S)), np.ones(T), s0)
    np.testing.assert_array_equal(st, s0)


def test_contraction_terms_symmetric_psd():
    rng = np.random.default_rng(16)
    S, D = 50, 12
    k = rng.standard_normal((S, D)) * O.key_scale(D, S)
    A, U = O.frame_terms(k, rng.standard_normal((S, D)), rng.random(S))
    np.testing.assert_allclose(A, A.T, atol=1e-15)
    assert np.linalg.eigvalsh(A).min() > -1e-14


def test_contraction_orientation_brute_force():
    """U[i, j] = sum_s beta_s v[s, i] k^[s, j] and A[i, j] likewise, by loops."""
    rng = np.random.default_rng(17)
    S, D = 3, 4
    k = rng.standard_normal((S, D))
    v = rng.standard_normal((S, D))
    beta = rng.random(S)
    A, U = O.frame_terms(k, v, beta)
    for i in range(D):
        for j in range(D):
            assert A[i, j] == pytest.approx(sum(beta[s] * k[s, i] * k[s, j] for s in range(S)))
            assert U[i, j] == pytest.approx(sum(beta[s] * v[s, i] * k[s, j] for s in range(S)))


def test_brute_force_explicit_transition_matrices():
    """S_t = S_{t-1} M_t + U_t with dense M_t and index loops (tiny sizes)."""
    rng = np.random.default_rng(18)
    T, S, D = 3, 4, 3
    q, k, v, beta, gamma = rand_case(rng, T, S, D)
    s0 = rng.standard_normal((D, D))
    out, st = O.frame_scan(q, k, v, beta, gamma, s0)
    c = 1 / np.sqrt(D * S)
    St = [[s0[i][j] for j in range(D)] for i in range(D)]
    for t in range(T):
        M = [[gamma[t] * ((1.0 if i == j else 0.0) -
                          sum(c * k[t, s, i] * beta[t, s] * c * k[t, s, j] for s in range(S)))
              for j in range(D)] for i in range(D)]
        U = [[sum(v[t, s, i] * beta[t, s] * c * k[t, s, j] for s in range(S))
              for j in range(D)] for i in range(D)]
        St = [[sum(St[i][m] * M[m][j] for m in range(D)) + U[i][j] for j in range(D)]
              for i in range(D)]
        for s in range(S):
            for i in range(D):
                assert out[t, s, i] == pytest.approx(sum(St[i][j] * q[t, s, j] for j in range(D)),
                                                     rel=1e-12, abs=1e-12)
    np.testing.assert_allclose(st, np.array(St), rtol=1e-12, atol=1e-12)


def test_non_expansive_when_trace_at_most_one():
    """'Jiayun's Blog' 2.1: tr(K^ beta K^^T) <= 1 implies ||M_t||_2 <= gamma_t."""
    rng = np.random.default_rng(19)
    checked = 0
    for _ in range(200):
        S, D = 16, 16
        k = rng.standard_normal((S, D)) * O.key_scale(D, S)
        beta = rng.random(S)
        A, _ = O.frame_terms(k, k, beta)
        if np.trace(A) > 1:
            continue
        g = 0.9 + 0.1 * rng.random()
        M = O.transition_matrix(k, beta, g)
        assert np.linalg.norm(M, 2) <= g * (1 + 1e-12)
        checked += 1
    assert checked > 100


def test_unscaled_keys_expand_scaled_keys_stay_bounded():
    """Without the 1/sqrt(D*S) scale the transition expands and the state
    blows up (the pages report NaN at step 16); with it the state stays bounded."""
    rng = np.random.default_rng(20)
    T, S, D = 1000, 16, 16
    k = rng.standard_normal((T, S, D))
    v = rng.standard_normal((T, S, D))
    beta = rng.random((T, S))
    gamma = 0.9 + 0.1 * rng.random(T)
    q = np.zeros((T, S, D))
    M_unscaled = O.transition_matrix(k[0], beta[0], gamma[0])
    assert np.linalg.norm(M_unscaled, 2) > 1.5
    with np.errstate(over="ignore", invalid="ignore"):
        _, st_bad = O.frame_scan(q[:40], k[:40], v[:40], beta[:40], gamma[:40], keys_scaled=True)
    assert not np.all(np.isfinite(st_bad)) or np.linalg.norm(st_bad) > 1e6
    _, st = O.frame_scan(q, k, v, beta, gamma)
    assert np.all(np.isfinite(st)) and np.linalg.norm(st) < 1e3


def test_linear_in_values_and_initial_state():
    rng = np.random.default_rng(21)
    T, S, D = 5, 6, 4
    q, k, v1, beta, gamma = rand_case(rng, T, S, D)
    v2 = rng.standard_normal((T, S, D))
    s1, s2 = rng.standard_normal((D, D)), rng.standard_normal((D, D))
    o1, t1 = O.frame_scan(q, k, v1, beta, gamma, s1)
    o2, t2 = O.frame_scan(q, k, v2, beta, gamma, s2)
    o3, t3 = O.frame_scan(q, k, 2 * v1 - v2, beta, gamma, 2 * s1 - s2)
    np.testing.assert_allclose(o3, 2 * o1 - o2, atol=1e-12)
    np.testing.assert_allclose(t3, 2 * t1 - t2, atol=1e-12)


# --- span composition ([HD] Context-Parallel section: exact) ------------------

@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("block", [0, 3])
@pytest.mark.parametrize("chunk", [1, 2, 3, 8, 11])
def test_chunked_equals_sequential(chunk, block, reverse):
    rng = np.random.default_rng(22)
    T, S, D = 11, 6, 5
    q, k, v, beta, gamma = rand_case(rng, T, S, D)
    s0 = rng.standard_normal((D, D))
    o_seq, st_seq = O.frame_scan(q, k, v, beta, gamma, s0, reverse=reverse, block=block)
    o_ch, st_ch = O.chunked_frame_scan(q, k, v, beta, gamma, s0, chunk=chunk,
                                       reverse=reverse, block=block)
    np.testing.assert_allclose(o_ch, o_seq, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(st_ch, st_seq, rtol=1e-11, atol=1e-12)


def test_composites_are_affine_maps():
    rng = np.random.default_rng(23)
    T, S, D = 4, 5, 3
    q, k, v, beta, gamma = rand_case(rng, T, S, D)
    C, Hm = O.chunk_composites(k, v, beta, gamma, list(range(T)), [False] * T)
    for _ in range(3):
        s0 = rng.standard_normal((D, D))
        _, st = O.frame_scan(q, k, v, beta, gamma, s0)
        np.testing.assert_allclose(s0 @ C + Hm, st, atol=1e-12)


# --- reverse scan and block reset (hyper.ai 方法; 实战指南 七) -----------------

def test_reverse_is_time_flipped_forward():
    rng = np.random.default_rng(24)
    T, S, D = 7, 4, 3
    q, k, v, beta, gamma = rand_case(rng, T, S, D)
    s0 = rng.standard_normal((D, D))
    o_r, st_r = O.frame_scan(q, k, v, beta, gamma, s0, reverse=True)
    o_f, st_f = O.frame_scan(q[::-1], k[::-1], v[::-1], beta[::-1], gamma[::-1], s0)
    np.testing.assert_allclose(o_r, o_f[::-1], atol=1e-13)
    np.testing.assert_allclose(st_r, st_f, atol=1e-13)


def test_reverse_block_reset_is_blockwise_flipped_forward():
    rng = np.random.default_rng(25)
    T, S, D, blk = 10, 4, 3, 3
    q, k, v, beta, gamma = rand_case(rng, T, S, D)
    o_r, _ = O.frame_scan(q, k, v, beta, gamma, reverse=True, block=blk)
    for b0 in range(0, T, blk):
        sl = slice(b0, min(b0 + blk, T))
        rs = slice(sl.stop - 1, b0 - 1 if b0 else None, -1)
        o_f, _ = O.frame_scan(q[rs], k[rs], v[rs], beta[rs], gamma[rs])
        np.testing.assert_allclose(o_r[sl], o_f[::-1], atol=1e-13)


def test_block_reset_isolates_blocks():
    rng = np.random.default_rng(26)
    T, S, D, blk = 9, 4, 3, 3
    q, k, v, beta, gamma = rand_case(rng, T, S, D)
    o1, _ = O.frame_scan(q, k, v, beta, gamma, reverse=True, block=blk)
    v2, k2 = v.copy(), k.copy()
    v2[6:] += 5.0
    k2[:3] *= -2.0
    o2, _ = O.frame_scan(q, k2, v2, beta, gamma, reverse=True, block=blk)
    np.testing.assert_allclose(o2[3:6], o1[3:6], atol=1e-13)
    assert not np.allclose(o2[6:], o1[6:])


def test_block_of_full_length_is_plain_reverse():
    rng = np.random.default_rng(27)
    T, S, D = 6, 3, 3
    q, k, v, beta, gamma = rand_case(rng, T, S, D)
    a, sa = O.frame_scan(q, k, v, beta, gamma, reverse=True, block=T)
    b, sb = O.frame_scan(q, k, v, beta, gamma, reverse=True)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(sa, sb)


def test_reset_positions():
    assert O.reset_before(O.scan_order(7, False), 3) == [False, False, False, True, False, False, True]
    # reverse over T=7: frames 6 | 5 4 3 | 2 1 0
    assert O.reset_before(O.scan_order(7, True), 3) == [False, True, False, False, True, False, False]


# --- prologue ----------------------------------------------------------------

def test_rmsnorm_unit_mean_square_and_weight():
    rng = np.random.default_rng(28)
    x = 3 * rng.standard_normal((10, 16))
    y = O.rmsnorm(x, np.ones(16), eps=0.0)
    np.testing.assert_allclose(np.mean(y * y, -1), 1.0, rtol=1e-13)
    w = rng.random(16)
    np.testing.assert_allclose(O.rmsnorm(x, w, eps=0.0), y * w, rtol=1e-13)


def test_relu_nonnegative():
    x = np.array([-2.0, -0.0, 0.5, 3.0])
    np.testing.assert_array_equal(O.relu(x), [0.0, 0.0, 0.5, 3.0])


def test_rope_orthogonal_identity_and_relative():
    rng = np.random.default_rng(29)
    W, Hh, D = 5, 4, 16
    S = W * Hh
    x = rng.standard_normal((S, D))
    y = O.rope2d(x, W)
    np.testing.assert_allclose(y[0], x[0], atol=0)                       # (0, 0) is identity
    pair = lambda z: z.reshape(S, D // 2, 2)
    np.testing.assert_allclose(np.linalg.norm(pair(y), axis=-1),
                               np.linalg.norm(pair(x), axis=-1), rtol=1e-13)
    # relative property: <R(p) a, R(p') b> depends only on p - p' (per axis)
    a, b = rng.standard_normal(D), rng.standard_normal(D)
    A = O.rope2d(np.tile(a, (S, 1)), W)
    B = O.rope2d(np.tile(b, (S, 1)), W)
    s1, s2 = 1 * W + 1, 2 * W + 3           # (y, x) = (1, 1), (2, 3)
    s3, s4 = 2 * W + 0, 3 * W + 2           # (2, 0), (3, 2): same offset (1, 2)
    assert A[s1] @ B[s2] == pytest.approx(A[s3] @ B[s4], rel=1e-12)
    # channel split: a pure x-shift leaves the first (y) half unchanged
    np.testing.assert_allclose(y[3, :D // 2], x[3, :D // 2], atol=0)
    np.testing.assert_allclose(y[2 * W, D // 2:], x[2 * W, D // 2:], atol=0)


def test_rope_frequency_of_first_pair():
    """Pair 0 of each half turns by exactly pos radians (theta_0 = 1)."""
    x = np.zeros((8, 8))
    x[:, 0] = 1.0
    x[:, 4] = 1.0
    y = O.rope2d(x, 4)
    s = 6                                    # (y, x) = (1, 2)
    assert y[s, 0] == pytest.approx(np.cos(1.0)) and y[s, 1] == pytest.approx(np.sin(1.0))
    assert y[s, 4] == pytest.approx(np.cos(2.0)) and y[s, 5] == pytest.approx(np.sin(2.0))


def test_rope_golden_pair_frequencies():
    """Hand-worked: at D = 8 pair 1 of each half turns by 10000^(-1/2) per
    position, so position 100 turns it by exactly 1 rad (derivation in the
    fixture); pins the frequency of every pair past the first."""
    g = json.load(open(os.path.join(GOLD, "rope2d_pair1.json")))
    for c in g["cases"]:
        x = np.zeros((c["S"], g["D"]))
        x[g["token"]] = g["x_in"]
        y = O.rope2d(x, c["grid_w"], g["base"])
        np.testing.assert_allclose(y[g["token"]], c["expected"], rtol=0, atol=1e-12)


def test_rmsnorm_golden_eps_inside_root():
    """Hand-worked: x = (3, 4), w = (2, 1/2), eps = 1/2 gives (6, 2)/sqrt(13)."""
    g = json.load(open(os.path.join(GOLD, "rmsnorm_eps.json")))
    y = O.rmsnorm(np.array(g["x"]), np.array(g["w"]), eps=g["eps"])
    np.testing.assert_allclose(y, g["expected"], rtol=0, atol=1e-14)


def test_prologue_order_and_key_scale():
    rng = np.random.default_rng(30)
    W, Hh, D = 4, 4, 16
    S = W * Hh
    q = rng.standard_normal((S, D))
    k = rng.standard_normal((S, D))
    wq, wk = 0.5 + rng.random(D), 0.5 + rng.random(D)
    qh, kh = O.qk_prologue(q, k, wq, wk, W)
    # RoPE is orthogonal, so norms equal those of the pre-RoPE vectors
    k_pre = O.key_scale(D, S) * O.relu(O.rmsnorm(k, wk))
    np.testing.assert_allclose(np.linalg.norm(kh, axis=-1), np.linalg.norm(k_pre, axis=-1), rtol=1e-12)
    assert np.all(np.abs(np.linalg.norm(qh, axis=-1) -
                         np.linalg.norm(O.relu(O.rmsnorm(q, wq)), axis=-1)) < 1e-12)
    np.testing.assert_allclose(kh[0], k_pre[0], atol=1e-15)    # token 0: no rotation


# --- camera encoding (UCPE) composed with the RoPE ----------------------------

def _rigid(rng):
    """A random rigid transform [[R, t], [0, 1]] (R a rotation)."""
    R, _ = np.linalg.qr(rng.standard_normal((3, 3)))
    if np.linalg.det(R) < 0:
        R[:, 0] *= -1
    T = np.eye(4)
    T[:3, :3] = R
    T[:3, 3] = 0.5 * rng.standard_normal(3)
    return T


def test_ucpe_golden():
    """Hand-worked (derivation in the fixture): a quarter turn with a shift on
    the camera block, RoPE on the other half."""
    g = json.load(open(os.path.join(GOLD, "ucpe_rope_d8.json")))
    x = np.zeros((g["S"], g["D"]))
    x[g["token"]] = g["x_in"]
    M = np.tile(np.eye(4), (g["S"], 1, 1))
    M[g["token"]] = g["M"]
    y = O.ucpe_rope(x, M, g["grid_w"], g["base"])
    np.testing.assert_allclose(y[g["token"]], g["expected"], rtol=0, atol=1e-12)


def test_ucpe_identity_is_rope_on_upper_half():
    rng = np.random.default_rng(40)
    W, Hh, D = 5, 3, 32
    S = W * Hh
    x = rng.standard_normal((S, D))
    y = O.ucpe_rope(x, np.tile(np.eye(4), (S, 1, 1)), W)
    np.testing.assert_array_equal(y[:, :D // 2], x[:, :D // 2])
    np.testing.assert_allclose(y[:, D // 2:], O.rope2d(x[:, D // 2:], W), rtol=0, atol=0)


def test_ucpe_scores_do_not_depend_on_the_world_frame():
    """Queries take D^T and keys D^-1 per token: every query-key product then
    depends on D_i D_j^-1 only, so moving the world frame (D -> D G^-1 for
    all tokens) leaves all products unchanged; a different world motion per
    token does not."""
    rng = np.random.default_rng(41)
    W, Hh, D = 4, 3, 16
    S = W * Hh
    q, k = rng.standard_normal((S, D)), rng.standard_normal((S, D))
    Dm = np.stack([_rigid(rng) for _ in range(S)])
    G = np.linalg.inv(_rigid(rng))

    def scores(Dm):
        qh = O.ucpe_rope(q, np.transpose(Dm, (0, 2, 1)), W)
        kh = O.ucpe_rope(k, np.linalg.inv(Dm), W)
        return qh @ kh.T

    base = scores(Dm)
    np.testing.assert_allclose(scores(Dm @ G), base, rtol=1e-10, atol=1e-10)
    Dm2 = Dm.copy()
    Dm2[3] = Dm2[3] @ G
    assert not np.allclose(scores(Dm2), base, atol=1e-6)


def test_ucpe_rotations_preserve_norms_and_prologue_uses_both_sides():
    rng = np.random.default_rng(42)
    W, Hh, D = 4, 2, 16
    S = W * Hh
    R = np.stack([_rigid(rng) for _ in range(S)])
    R[:, :3, 3] = 0.0                       # pure rotations: M^T = M^-1
    x = rng.standard_normal((S, D))
    y = O.ucpe_rope(x, R, W)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)
    q, k = rng.standard_normal((S, D)), rng.standard_normal((S, D))
    w = 0.5 + rng.random(D)
    Mq, Mk = np.transpose(R, (0, 2, 1)), np.linalg.inv(R)
    qh, kh = O.qk_prologue(q, k, w, w, W, ucpe=(Mq, Mk))
    np.testing.assert_allclose(qh, O.ucpe_rope(O.relu(O.rmsnorm(q, w)), Mq, W), rtol=1e-13)
    np.testing.assert_allclose(kh, O.ucpe_rope(O.key_scale(D, S) * O.relu(O.rmsnorm(k, w)), Mk, W),
                               rtol=1e-13)


def test_ucpe_blocks_by_index_loops():
    """Brute force at D = 16 (two camera blocks): out[4b + i] = sum_j M[i][j] x[4b + j]."""
    rng = np.random.default_rng(45)
    S, D = 6, 16
    x, M = rng.standard_normal((S, D)), rng.standard_normal((S, 4, 4))
    y = O.ucpe_rope(x, M, 3)
    for s_ in range(S):
        for b in range(D // 8):
            for i in range(4):
                acc = 0.0
                for j in range(4):
                    acc += M[s_][i][j] * x[s_][4 * b + j]
                assert abs(y[s_][4 * b + i] - acc) < 1e-12
