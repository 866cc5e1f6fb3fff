"""Float64 CPU oracle of the frame-wise Gated DeltaNet (GDN) frame scan.

TEST INFRASTRUCTURE ONLY (see the package docstring): nothing on the product
path imports this module, and it imports nothing from the product path.

Sources, cited by page title and section:

[HD] "SANA-WM：2.6B 参数分布式 Diffusion Transformer 实现消费级 GPU 分钟级 720p
     视频生成" (blog.hotdry.top).
     Section "混合线性注意力：长上下文的内存破局点": the frame-wise recurrence
     S_t = S_{t-1} M_t + U_t with M_t = gamma_t (I - K^_t beta_t K^_t^T) and
     U_t = V_t beta_t K^_t^T, a D x D state per frame, beta per token, and the
     key scale 1/sqrt(D*S).
     Section "显存分片：Context-Parallel 的工程实现": per-span composites C_p, H_p
     with S_end = S_start C_p + H_p, stated to be exact; the fused prologue
     order RMSNorm -> ReLU -> key scale -> UCPE/RoPE -> scan.
[JY] "Jiayun's Blog", post on NVIDIA SANA-WM (xiejiayun.github.io),
     section 2.1 "Frame-wise GDN": the token-wise GDN step
     S_i = gamma_i S_{i-1} + (v_i - gamma_i S_{i-1} k^_i) beta_i k^_i^T
     (subscripts restored, the extraction dropped them), the frame-wise form,
     S = 80 x 45 = 3600, and tr(K^ beta K^^T) <= 1  =>  ||M_t||_2 <= gamma_t.
[HA] hyper.ai summary of the SANA-WM paper (hyper.ai/cn/papers/2605.15178),
     section "方法": the chunk-causal variant resets the reverse-time scan at
     chunk boundaries.
[TR] "SANA-WM 世界模型实战指南" (trdm.cn), section 七 (Stage-1 Teacher 训练):
     attention types BidirectionalGDNTriton / ChunkCausalGDNTriton and
     chunk_size: 3.

Layout: per (b, h) the frame tensors are [T, S, D] (token-major, D last),
beta is [T, S], gamma is [T], the state is [D, D] with rows indexing the value
channel and columns the key channel (the shape of V beta K^^T in [HD]).

Readings where the pages are silent (each is listed in the design notes):
  R1  the readout is O_t = S_t Q_t with the post-update state S_t, i.e. for
      token s: o_s = S_t q_s; no query scale.
  R4  the key scale uses the frame's full token count S in both A_t and U_t.
  R5  the reverse scan is the time-mirrored recurrence, inclusive of frame t,
      returned as its own output.
  R6  blocks for the chunk reset are floor(t / block) counted from t = 0 in
      both directions; the state is zeroed on entering a new block in scan
      order; state_in seeds only the first block in scan order.
  R8-R10  RMSNorm over D with eps inside the root, then ReLU, then (keys
      only) the key scale, then a 2-D spatial RoPE: token s = y*W + x; channels
      [0, D/2) rotate with y, [D/2, D) with x; inside each half the pairs
      (2i, 2i+1), i < D/4, turn by pos * base^(-2i/(D/2)).
  R20 camera encoding (UCPE): the caller gives each token's 4 x 4 matrices,
      D_{t,s}^T for queries and D_{t,s}^-1 for keys (D_{t,s}: world -> the
      token's ray-local frame), shared by all heads; a query-key product then
      depends on D_i D_j^-1 only, not on the world frame.
  R21 "combined orthogonally with RoPE": on separate channels; the camera
      blocks of 4 take [0, D/2), the 2-D RoPE (R10 on D/2 channels) [D/2, D).

Pins (tests/test_oracle_pins.py) and their status per function:
  frame_scan / gdn_frame_scan   pinned (token-wise reduction, delta-rule
                                retrieval, closed-form geometric cases, golden
                                fixtures, invariants, brute force)
  chunked_frame_scan            pinned (equals frame_scan; exactness per [HD])
  readout (inside frame_scan)   definition pinned by reading R1 only: parity
                                with the pages' own readout is unpinned.
  qk_prologue                   pinned by invariants (mean square, sign,
                                orthogonality, identity, relative phase) and
                                by hand-worked fixtures of its constants
                                (eps inside the root and the weight after the
                                normalisation; every pair's frequency, the
                                axis split, the pair layout and the turn
                                direction). The constants themselves are
                                readings R8-R10: the pages do not fix them.
  ucpe_rope                     pinned by a hand-worked fixture (a quarter
                                turn of one block plus RoPE on the rest),
                                the identity transform reducing to rope2d on
                                the upper half, invariance of every
                                query-key product under a change of world
                                frame, and norm preservation for rotations.
                                The transform's source (ray-local frames
                                from poses) is the caller's, readings
                                R20-R21.
  frame_scan_bwd                the pages print no backward; this is the
                                adjoint of frame_scan derived by reverse-mode
                                differentiation, pinned by central finite
                                differences of frame_scan for every input
                                (tests/test_oracle_backward.py).
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "key_scale",
    "frame_terms",
    "transition_matrix",
    "scan_order",
    "reset_before",
    "frame_scan",
    "gdn_frame_scan",
    "chunk_composites",
    "chunked_frame_scan",
    "token_wise_gdn",
    "rmsnorm",
    "ucpe_rope",
    "relu",
    "rope2d",
    "qk_prologue",
    "frame_scan_bwd",
]


# ---------------------------------------------------------------------------
# Frame-wise GDN ([HD] 混合线性注意力; [JY] 2.1)
# ---------------------------------------------------------------------------

def key_scale(D: int, S: int) -> float:
    """The key scale 1/sqrt(D*S) of [HD] and [JY] 2.1 (reading R4: S is the
    number of spatial tokens of one frame)."""
    return 1.0 / np.sqrt(float(D) * float(S))


def frame_terms(k_hat: np.ndarray, v: np.ndarray, beta: np.ndarray):
    """A_t = K^_t beta_t K^_t^T and U_t = V_t beta_t K^_t^T for one frame.

    k_hat, v: [S, D] (keys already scaled); beta: [S]. With the keys stored
    token-major, the page's K^_t (D x S) is k_hat^T, so
    A = k_hat^T diag(beta) k_hat and U = v^T diag(beta) k_hat, both D x D.
    """
    bk = beta[:, None] * k_hat
    A = k_hat.T @ bk
    U = v.T @ bk
    return A, U


def transition_matrix(k_hat: np.ndarray, beta: np.ndarray, gamma: float):
    """M_t = gamma_t (I - K^_t beta_t K^_t^T), written out as a dense matrix."""
    D = k_hat.shape[1]
    A, _ = frame_terms(k_hat, np.zeros_like(k_hat), beta)
    return gamma * (np.eye(D) - A)


def scan_order(T: int, reverse: bool):
    """Frame indices in scan order (reading R5 for the reverse direction)."""
    return list(range(T - 1, -1, -1)) if reverse else list(range(T))


def reset_before(order, block: int):
    """For each position j of the scan order: True when the carried state is
    zeroed before frame order[j] (reading R6: a new block, floor(t/block), is
    entered; never before the first processed frame)."""
    out = []
    for j, t in enumerate(order):
        out.append(bool(block) and j > 0 and (t // block) != (order[j - 1] // block))
    return out


def frame_scan(q, k, v, beta, gamma, state_in=None, *, reverse=False, block=0,
               keys_scaled=False):
    """The sequential frame-wise GDN scan for one (b, h), in float64.

    q, k, v: [T, S, D]; beta: [T, S]; gamma: [T]; state_in: [D, D] or None.
    For each frame t in scan order ([HD] 混合线性注意力):
        K^ = k / sqrt(D*S)             (skipped when keys_scaled)
        A  = K^^T diag(beta) K^,  U = V^T diag(beta) K^
        S  = gamma_t (S - S A) + U     (= S M_t + U_t)
        O_t = Q_t S^T                  (o_s = S q_s; reading R1)
    Returns (O [T, S, D], state after the last processed frame [D, D]).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    beta = np.asarray(beta, np.float64)
    gamma = np.asarray(gamma, np.float64)
    T, S, D = q.shape
    c = 1.0 if keys_scaled else key_scale(D, S)
    St = np.zeros((D, D)) if state_in is None else np.array(state_in, np.float64)
    O = np.empty((T, S, D))
    order = scan_order(T, reverse)
    resets = reset_before(order, block)
    for t, rst in zip(order, resets):
        if rst:
            St = np.zeros((D, D))
        A, U = frame_terms(c * k[t], v[t], beta[t])
        St = gamma[t] * (St - St @ A) + U
        O[t] = q[t] @ St.T
    return O, St


def gdn_frame_scan(q, k, v, beta, gamma, state_in=None, *, reverse=False,
                   block=0, keys_scaled=False):
    """frame_scan over a batch: q, k, v [B, H, T, S, D]; beta [B, H, T, S];
    gamma [B, H, T]; state_in [B, H, D, D] or None. Returns (O, state_out)."""
    B, H, T, S, D = np.shape(q)
    O = np.empty((B, H, T, S, D))
    Sout = np.empty((B, H, D, D))
    for b in range(B):
        for h in range(H):
            s0 = None if state_in is None else state_in[b][h]
            O[b, h], Sout[b, h] = frame_scan(
                q[b][h], k[b][h], v[b][h], beta[b][h], gamma[b][h], s0,
                reverse=reverse, block=block, keys_scaled=keys_scaled)
    return O, Sout


# ---------------------------------------------------------------------------
# Affine span composition ([HD] 显存分片：Context-Parallel 的工程实现)
# ---------------------------------------------------------------------------

def chunk_composites(k, v, beta, gamma, frames, resets, *, keys_scaled=False):
    """Transition composite C and input composite H of one span of frames.

    frames: frame indices in scan order; resets: per frame, whether the carried
    state is zeroed before it. Starting from C = I, H = 0, each frame applies
    the same affine step the state takes: (C, H) <- (C M_t, H M_t + U_t), and a
    reset replaces (C, H) by (0, 0) first. Then for any S_start the span maps
    S_start to S_start C + H ([HD]: S_end = S_start C_p + H_p).
    """
    T, S, D = np.shape(k)
    c = 1.0 if keys_scaled else key_scale(D, S)
    C = np.eye(D)
    Hm = np.zeros((D, D))
    for t, rst in zip(frames, resets):
        if rst:
            C = np.zeros((D, D))
            Hm = np.zeros((D, D))
        A, U = frame_terms(c * np.asarray(k[t], np.float64),
                           np.asarray(v[t], np.float64),
                           np.asarray(beta[t], np.float64))
        M = gamma[t] * (np.eye(D) - A)
        C = C @ M
        Hm = Hm @ M + U
    return C, Hm


def chunked_frame_scan(q, k, v, beta, gamma, state_in=None, *, chunk=8,
                       reverse=False, block=0, keys_scaled=False):
    """The same scan computed span by span ([HD] Context-Parallel section):
    per span of `chunk` frames (in scan order) the composites (C_p, H_p); a
    prefix S_start^(p+1) = S_start^(p) C_p + H_p; then each span replays its
    frames from its exact start state. Equal to frame_scan up to rounding."""
    q = np.asarray(q, np.float64)
    T, S, D = q.shape
    c = 1.0 if keys_scaled else key_scale(D, S)
    order = scan_order(T, reverse)
    resets = reset_before(order, block)
    spans = [list(range(p, min(p + chunk, T))) for p in range(0, T, chunk)]
    comps = [chunk_composites(k, v, beta, gamma, [order[j] for j in sp],
                              [resets[j] for j in sp], keys_scaled=keys_scaled)
             for sp in spans]
    starts = []
    St = np.zeros((D, D)) if state_in is None else np.array(state_in, np.float64)
    for C, Hm in comps:
        starts.append(St)
        St = St @ C + Hm
    state_out = St
    O = np.empty((T, S, D))
    for sp, St in zip(spans, starts):
        for j in sp:
            t = order[j]
            if resets[j]:
                St = np.zeros((D, D))
            A, U = frame_terms(c * np.asarray(k[t], np.float64),
                               np.asarray(v[t], np.float64),
                               np.asarray(beta[t], np.float64))
            St = gamma[t] * (St - St @ A) + U
            O[t] = q[t] @ St.T
    return O, state_out


# ---------------------------------------------------------------------------
# Token-wise GDN ([JY] 2.1), the special case S = 1
# ---------------------------------------------------------------------------

def token_wise_gdn(q, k_hat, v, beta, gamma, state_in=None):
    """Original token-wise Gated DeltaNet, one token per step ([JY] 2.1):
        S_i = gamma_i S_{i-1} + (v_i - gamma_i S_{i-1} k^_i) beta_i k^_i^T
        o_i = S_i q_i
    q, k_hat, v: [N, D]; beta, gamma: [N]. Returns (o [N, D], S_N)."""
    N, D = np.shape(q)
    St = np.zeros((D, D)) if state_in is None else np.array(state_in, np.float64)
    o = np.empty((N, D))
    for i in range(N):
        kk = np.asarray(k_hat[i], np.float64)
        pred = gamma[i] * (St @ kk)
        St = gamma[i] * St + beta[i] * np.outer(np.asarray(v[i], np.float64) - pred, kk)
        o[i] = St @ np.asarray(q[i], np.float64)
    return o, St


# ---------------------------------------------------------------------------
# Prologue ([HD] 显存分片 section: RMSNorm, ReLU, key scale, RoPE prep)
# ---------------------------------------------------------------------------

def rmsnorm(x, w, eps=1e-6):
    """x / sqrt(mean(x^2 over D) + eps) * w (reading R8)."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(w, np.float64)


def relu(x):
    return np.maximum(np.asarray(x, np.float64), 0.0)


def rope2d(x, grid_w, base=10000.0):
    """2-D spatial rotary embedding on the last two axes [S, D] (reading R10).

    Token s sits at (y, x) = divmod(s, grid_w). Channels [0, D/2) turn with y,
    channels [D/2, D) with x; in each half the pair (2i, 2i+1), i < D/4, turns
    by phi = pos * base^(-2i/(D/2)): (a, b) -> (a cos phi - b sin phi,
    a sin phi + b cos phi)."""
    x = np.array(x, np.float64)
    S, D = x.shape[-2], x.shape[-1]
    half = D // 2
    s = np.arange(S)
    pos_y, pos_x = s // grid_w, s % grid_w
    out = x.copy()
    for i in range(D // 4):
        theta = base ** (-2.0 * i / half)
        for off, pos in ((0, pos_y), (half, pos_x)):
            phi = pos * theta
            cs, sn = np.cos(phi), np.sin(phi)
            a = x[..., off + 2 * i]
            b = x[..., off + 2 * i + 1]
            out[..., off + 2 * i] = a * cs - b * sn
            out[..., off + 2 * i + 1] = a * sn + b * cs
    return out


def ucpe_rope(x, M, grid_w, base=10000.0):
    """Camera encoding composed with the 2-D RoPE on separate channels
    ([HD] section 双分支相机控制: a per-token homogeneous transform D_{t,s}
    from world to the token's ray-local frame, combined orthogonally with
    RoPE; [JY] 2.3; readings R20-R21).

    x: [..., S, D]; M: [..., S, 4, 4], the matrix applied to this side's
    tokens (queries take D_{t,s}^T, keys D_{t,s}^-1, so that a query-key
    product sees D_i D_j^-1 only). Channels [0, D/2) form D/8 blocks of 4
    (block b = channels 4b .. 4b+3); each block of token s becomes M[s] times
    it. Channels [D/2, D) get rope2d as a vector of D/2 channels (its y half
    first, then its x half)."""
    x = np.array(x, np.float64)
    M = np.asarray(M, np.float64)
    D = x.shape[-1]
    h = D // 2
    out = x.copy()
    for b in range(h // 4):
        blk = x[..., 4 * b:4 * b + 4]
        out[..., 4 * b:4 * b + 4] = np.einsum("...ij,...j->...i", M, blk)
    out[..., h:] = rope2d(x[..., h:], grid_w, base)
    return out


def qk_prologue(q_raw, k_raw, w_q, w_k, grid_w, *, eps=1e-6, base=10000.0, ucpe=None):
    """Prologue in the pages' order ([HD] 显存分片 section; readings R8-R10):
    RMSNorm -> ReLU -> key scale 1/sqrt(D*S) (keys only) -> 2-D RoPE, or,
    with ucpe = (M_q, M_k) ([..., S, 4, 4] each), -> ucpe_rope.
    q_raw, k_raw: [..., S, D]. Returns (q^, k^); k^ carries the key scale."""
    S, D = np.shape(q_raw)[-2], np.shape(q_raw)[-1]
    qn = relu(rmsnorm(q_raw, w_q, eps))
    kn = key_scale(D, S) * relu(rmsnorm(k_raw, w_k, eps))
    if ucpe is None:
        return rope2d(qn, grid_w, base), rope2d(kn, grid_w, base)
    return ucpe_rope(qn, ucpe[0], grid_w, base), ucpe_rope(kn, ucpe[1], grid_w, base)


# ---------------------------------------------------------------------------
# Backward of the frame scan (adjoint; the pages give no formula)
# ---------------------------------------------------------------------------

def frame_scan_bwd(q, k, v, beta, gamma, state_in, d_out, d_state_out=None, *,
                   reverse=False, block=0, keys_scaled=False):
    """Gradients of a scalar loss through frame_scan for one (b, h), float64.

    Given d_out = dL/dO [T, S, D] and d_state_out = dL/d(state after the last
    processed frame) [D, D] (or None), returns
    (dq, dk, dv, dbeta, dgamma, d_state_in) with the shapes of the inputs
    (d_state_in is zeros when state_in is None).

    Derivation (reverse mode over the scan order j = 0..T-1, frame t_j):
        X_j = g_j (X'_{j-1} - X'_{j-1} A_j) + U_j,  X'_{j-1} = X_{j-1}, or 0
              after a reset, or state_in at j = 0;   O_{t_j} = Q_{t_j} X_j^T
    The total gradient reaching X_j is
        G_j = dO_{t_j}^T Q_{t_j} + [G_{j+1} M_{j+1}^T unless j+1 resets]
              (+ d_state_out at the last j),   M = g (I - A),
    and for frame j:  dU = G_j,  dM = X'_{j-1}^T G_j,
        dA = -g_j dM,  dg_j = <dM, I - A_j>,  dQ_t = dO_t X_j.
    Through A = K^^T diag(beta) K^ and U = V^T diag(beta) K^ (rows k^_s, v_s):
        dk^_s = beta_s ((dA + dA^T) k^_s + dU^T v_s)
        dv_s  = beta_s dU k^_s
        dbeta_s = k^_s . dA k^_s + v_s . dU k^_s
    and dk = c dk^ (c = 1/sqrt(D S) unless keys_scaled). d_state_in is the
    carry G_0 M_0^T into the state entering the first frame.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    beta = np.asarray(beta, np.float64)
    gamma = np.asarray(gamma, np.float64)
    d_out = np.asarray(d_out, np.float64)
    T, S, D = q.shape
    c = 1.0 if keys_scaled else key_scale(D, S)
    order = scan_order(T, reverse)
    resets = reset_before(order, block)
    s0 = np.zeros((D, D)) if state_in is None else np.array(state_in, np.float64)
    # forward, keeping the state entering each frame (after any reset) and A, U
    prev, As, states = [], [], []
    X = s0
    for t, rst in zip(order, resets):
        if rst:
            X = np.zeros((D, D))
        A, U = frame_terms(c * k[t], v[t], beta[t])
        prev.append(X)  # state entering frame j (after any reset)
        As.append(A)
        X = gamma[t] * (X - X @ A) + U
        states.append(X)  # state after frame j
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dbeta = np.zeros_like(beta)
    dgamma = np.zeros_like(gamma)
    G_next = None
    d_s0 = np.zeros((D, D))
    I = np.eye(D)
    for j in range(T - 1, -1, -1):
        t = order[j]
        G = d_out[t].T @ q[t]
        if j == T - 1 and d_state_out is not None:
            G = G + np.asarray(d_state_out, np.float64)
        if G_next is not None:
            G = G + G_next
        dq[t] = d_out[t] @ states[j]
        A = As[j]
        dM = prev[j].T @ G
        dA = -gamma[t] * dM
        dgamma[t] = np.sum(dM * (I - A))
        dU = G
        kh = c * k[t]
        sym = dA + dA.T
        dkh = beta[t][:, None] * (kh @ sym.T + v[t] @ dU)
        dv[t] = beta[t][:, None] * (kh @ dU.T)
        dbeta[t] = np.einsum("sd,sd->s", kh, kh @ dA.T) + np.einsum("sd,sd->s", v[t] @ dU, kh)
        dk[t] = c * dkh
        carry = G @ (gamma[t] * (I - A)).T  # gradient reaching the state entering frame j
        if resets[j]:
            G_next = None
        elif j == 0:
            d_s0 = carry
        else:
            G_next = carry
    return dq, dk, dv, dbeta, dgamma, d_s0
