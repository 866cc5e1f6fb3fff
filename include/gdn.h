/*
 * gdn.h — C ABI of libgdnscan.so, a B200 (sm_100a) implementation of the
 * frame-wise Gated DeltaNet (GDN) frame scan.
 *
 * What it computes. For every batch b, head h and latent frame t, with the S
 * spatial tokens of the frame stored token-major (Q_t, K_t, V_t are S x D):
 *
 *     K^_t = K_t / sqrt(D*S)                       key scale
 *     A_t  = K^_t^T diag(beta_t) K^_t              D x D, symmetric PSD
 *     U_t  = V_t^T  diag(beta_t) K^_t              D x D
 *     S_t  = gamma_t (S_{t-1} - S_{t-1} A_t) + U_t   (= S_{t-1} M_t + U_t)
 *     O_t  = Q_t S_t^T                             token s: o_s = S_t q_s
 *
 * Sources (web pages on SANA-WM, cited by title and section):
 *  - "SANA-WM：2.6B 参数分布式 Diffusion Transformer 实现消费级 GPU 分钟级 720p
 *    视频生成" (blog.hotdry.top), section "混合线性注意力：长上下文的内存破局点":
 *    the recurrence S_t = S_{t-1} M_t + U_t, M_t = gamma_t (I - K^ beta K^^T),
 *    U_t = V beta K^^T, one D x D state update per frame, beta per token, and
 *    the key scale 1/sqrt(D*S). Section "显存分片：Context-Parallel 的工程实现":
 *    S_end = S_start C_p + H_p per span of frames (used here to run time
 *    chunks in parallel on one GPU), and the fused prologue order RMSNorm ->
 *    ReLU -> key scale -> RoPE -> scan.
 *  - "Jiayun's Blog", post on SANA-WM, section 2.1: the same frame-wise form,
 *    S = 80 x 45 = 3600 tokens per 720p latent frame.
 *  - hyper.ai summary of the SANA-WM paper, section "方法": the chunk-causal
 *    variant resets the reverse-time scan at chunk boundaries.
 *  - "SANA-WM 世界模型实战指南" (trdm.cn), section 七: chunk_size: 3.
 * The readout O_t = S_t Q_t with the post-update state is not written out on
 * the pages; it is the plain reading, matching token-wise GDN's o_i = S_i q_i.
 *
 * Conventions shared by every entry point.
 *  - Layouts: q, k, v, out are [B, H, T, S, D] contiguous (D innermost),
 *    bf16 when GDN_BF16 is set, else fp32; beta is [B, H, T, S] fp32; gamma
 *    is [B, H, T] fp32; states are [B, H, D, D] fp32 row-major, row = value
 *    channel, column = key channel.
 *  - All pointers are DEVICE pointers, owned by the caller, 16-byte aligned.
 *    Outputs must not alias inputs.
 *  - Shapes: D in {16, 32, 64, 128, 256}; S >= 1; T >= 1; B, H >= 1.
 *  - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream); no entry point synchronises the host except
 *    gdn_check_device_status.
 *  - Execution: the library is built for sm_100a (B200) only. bf16 inputs
 *    at D in {64, 128, 256} run on the tensor cores (tcgen05, TMA); at
 *    D = 256 the contraction and the readout launch clusters of two CTAs
 *    that share one MMA, and a device that cannot hold such a cluster makes
 *    those calls return GDN_ERR_CUDA. fp32 inputs, D in {16, 32} and
 *    GDN_FORCE_SIMT run on CUDA cores.
 *  - Errors: argument errors return GDN_ERR_INVALID / GDN_ERR_UNSUPPORTED
 *    before anything is launched; a failed launch returns GDN_ERR_CUDA; a
 *    device-side bounded wait that ran out is reported by
 *    gdn_check_device_status as GDN_ERR_TIMEOUT. gdn_last_error() gives a
 *    one-line description of the last failure on the calling host thread.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

typedef struct CUstream_st* gdn_stream_t; /* identical to cudaStream_t */

enum {
  GDN_OK = 0,
  GDN_ERR_INVALID = -1,     /* null/misaligned pointer, bad size or flag combination */
  GDN_ERR_UNSUPPORTED = -2, /* D outside {16,32,64,128,256}, or sizes past index limits */
  GDN_ERR_CUDA = -3,        /* a CUDA runtime call or launch failed */
  GDN_ERR_TIMEOUT = -4,     /* a device-side bounded wait expired */
  GDN_ERR_WORKSPACE = -5    /* workspace missing or smaller than gdn_workspace_bytes */
};

/* flags */
#define GDN_BF16 0x1u           /* q/k/v/out are bf16, else fp32 */
#define GDN_REVERSE 0x2u        /* reverse-time scan: frames T-1 .. 0 */
#define GDN_BLOCK_RESET 0x4u    /* zero the state on entering each block (scan order) */
#define GDN_SEQUENTIAL 0x8u     /* one chain over T, no span composition */
#define GDN_FUSED_PROLOGUE 0x10u /* _ex only: q, k are raw; apply the prologue */
#define GDN_KEYS_SCALED 0x20u   /* k already carries 1/sqrt(D*S): do not scale again */
#define GDN_FORCE_SIMT 0x40u    /* use the CUDA-core kernels even where tensor-core ones exist */
#define GDN_BIDIR 0x80u         /* _ex only: forward scan -> out, reverse scan -> out_rev */
#define GDN_FUSED_REPLAY 0x1000000u /* tensor-core path: replay each span inside the readout
                                       kernel instead of storing S_t (spans/blocks, no prologue) */
#define GDN_CHUNKED 0x2000000u  /* run the span-composed (chunk-parallel) plan */
#define GDN_REV_STATE_IN 0x8000000u /* _ex with GDN_BIDIR: the reverse scan starts from
                                       state_in_rev (NULL = zeros) instead of state_in */
#define GDN_NO_OVERLAP 0x4000000u /* run the sequential chains as their own launch after
                                     the contraction instead of alongside it */
#define GDN_UCPE 0x20000000u     /* _ex with GDN_FUSED_PROLOGUE: camera encoding on
                                   channels [0, D/2) (ucpe_q, ucpe_k), RoPE on [D/2, D);
                                   see gdn_qk_prologue_ucpe */
#define GDN_SAVE_FOR_BACKWARD 0x10000000u /* _ex: leave the A_t operand images and the
                                     states in the workspace for gdn_frame_scan_bwd's
                                     saved_workspace (otherwise the plan with the chains
                                     alongside the contraction lets the A_t images go
                                     once read, so they never cost an HBM write) */
#define GDN_BLOCK(f) (((f) >> 8) & 0xffu)  /* reset block length; 0 means 3 */
#define GDN_CHUNK(f) (((f) >> 16) & 0xffu) /* time-chunk length; 0 means 8 */
#define GDN_MAKE_BLOCK(n) ((((unsigned)(n)) & 0xffu) << 8)
#define GDN_MAKE_CHUNK(n) ((((unsigned)(n)) & 0xffu) << 16)

/*
 * gdn_frame_scan_fwd — the whole frame scan for [B, H] heads over T frames.
 *
 *   q, k, v     [B,H,T,S,D]  bf16 (GDN_BF16) or fp32, device
 *   beta        [B,H,T,S]    fp32 per-token update gate
 *   gamma       [B,H,T]      fp32 per-frame decay
 *   state_in    [B,H,D,D]    fp32 state entering the first frame in scan
 *                            order; NULL means zeros. With GDN_BLOCK_RESET it
 *                            seeds only the first block in scan order.
 *   out         [B,H,T,S,D]  same dtype as q: O_t = Q_t S_t^T
 *   state_out   [B,H,D,D]    fp32 state after the last frame in scan order
 *                            (frame T-1 forward, frame 0 reversed); NULL = not written
 *   flags       GDN_BF16 | GDN_REVERSE | GDN_BLOCK_RESET | GDN_SEQUENTIAL |
 *               GDN_CHUNKED | GDN_NO_OVERLAP | GDN_KEYS_SCALED |
 *               GDN_FORCE_SIMT | GDN_FUSED_REPLAY | GDN_MAKE_BLOCK(n) |
 *               GDN_MAKE_CHUNK(n)
 *
 * Blocks for GDN_BLOCK_RESET are floor(t / block) counted from t = 0 in both
 * directions.
 *
 * Plans (all equal up to rounding). GDN_SEQUENTIAL: one chain of the
 * recurrence per head over all T frames. GDN_CHUNKED: time chunks composed
 * through S_end = S_start C_p + H_p (SANA-WM blog, Context-Parallel section),
 * run in parallel, then replayed. Neither flag: the sequential plan where it
 * can run alongside the contraction, else the chunked plan. Alongside means
 * one cooperative launch in which a few CTAs run the chains (one per head and
 * direction) while the rest compute A_t, U_t frame by frame, so the
 * latency-bound chains hide under the bandwidth-bound contraction. It needs
 * the tensor-core path (bf16, sm_100a), D = 128, at most a quarter of the
 * GPU's SMs in chains (B*H <= 37 on a 148-SM B200; 2*B*H for GDN_BIDIR, which
 * also needs GDN_BLOCK_RESET), and no GDN_FUSED_REPLAY. GDN_NO_OVERLAP turns
 * it off. With very few frame-heads (B*H*T at most a quarter of the SMs, at
 * least 193 tokens per frame) the contraction instead cuts each frame-head's
 * tokens over several CTAs and the chains follow in their own launch.
 * Scratch comes from a stream-ordered allocation (cudaMallocAsync)
 * made and freed inside the call; use gdn_frame_scan_fwd_ex to pass your own.
 * Returns GDN_OK or a negative status.
 */
GDN_API int gdn_frame_scan_fwd(const void* q, const void* k, const void* v, const float* beta,
                       const float* gamma, const float* state_in, void* out, float* state_out,
                       int B, int H, int T, int S, int D, unsigned flags, gdn_stream_t stream);

/*
 * gdn_qk_prologue — the per-token prologue ahead of the scan, in the pages'
 * order (SANA-WM blog, Context-Parallel section: RMSNorm -> ReLU -> key scale
 * -> RoPE), on raw q and k:
 *     x <- x / sqrt(mean_D(x^2) + eps) * w        (w_q for q, w_k for k)
 *     x <- max(x, 0)
 *     k <- k / sqrt(D*S)                           (keys only; S = grid_h*grid_w)
 *     x <- RoPE2D(x): token s at (y, x) = (s / grid_w, s % grid_w); channels
 *          [0, D/2) turn with y, [D/2, D) with x; pair (2i, 2i+1) of a half,
 *          i < D/4, turns by pos * rope_base^(-2i/(D/2)).
 *   q_raw, k_raw    [B,H,T,S,D] bf16 or fp32 (GDN_BF16), device
 *   w_q, w_k        [D] fp32
 *   q_out, k_out    [B,H,T,S,D] same dtype; k_out carries the key scale, so a
 *                   following gdn_frame_scan_fwd takes GDN_KEYS_SCALED.
 * Only GDN_BF16 is read from flags. Returns GDN_OK or a negative status.
 */
GDN_API int gdn_qk_prologue(const void* q_raw, const void* k_raw, const float* w_q, const float* w_k,
                    void* q_out, void* k_out, int B, int H, int T, int grid_h, int grid_w, int D,
                    float eps, float rope_base, unsigned flags, gdn_stream_t stream);

/*
 * gdn_qk_prologue_ucpe — the prologue with the camera encoding (SANA-WM blog,
 * section 双分支相机控制：从粗到细的 6-DoF 轨迹: for every token a homogeneous
 * transform D_{t,s} from world coordinates into the token's ray-local frame,
 * combined orthogonally with the RoPE; "Jiayun's Blog", section 2.3). The
 * pages do not say how the two are combined or how D enters the attention;
 * readings: they act on separate channels, and queries take D^T, keys D^-1,
 * so that a query-key product depends only on D_i D_j^-1 (not on the world
 * frame). Per token, after RMSNorm, ReLU and (keys) the key scale:
 *     channels [0, D/2): block b (channels 4b .. 4b+3) <- M block b, with M
 *                        = ucpe_q[b,t,s] for q and ucpe_k[b,t,s] for k;
 *     channels [D/2, D): the 2-D RoPE of gdn_qk_prologue applied to them as
 *                        a vector of D/2 channels (its first half turns with
 *                        y, its second half with x).
 *   ucpe_q, ucpe_k  [B,T,S,4,4] fp32 row-major device arrays, 16-byte aligned,
 *                   shared by all heads (for pure rotations D^T = D^-1: pass
 *                   the same array twice). Computing D_{t,s} from camera
 *                   poses and intrinsics is the caller's.
 * Other arguments, outputs and errors as gdn_qk_prologue. */
GDN_API int gdn_qk_prologue_ucpe(const void* q_raw, const void* k_raw, const float* w_q,
                                 const float* w_k, const float* ucpe_q, const float* ucpe_k,
                                 void* q_out, void* k_out, int B, int H, int T, int grid_h,
                                 int grid_w, int D, float eps, float rope_base, unsigned flags,
                                 gdn_stream_t stream);

/* Everything gdn_frame_scan_fwd takes, plus the prologue, the second
 * direction and caller-owned scratch. Zero-initialise and fill. */
typedef struct gdn_params {
  const void* q;          /* [B,H,T,S,D]; raw when GDN_FUSED_PROLOGUE */
  const void* k;          /* [B,H,T,S,D]; raw when GDN_FUSED_PROLOGUE */
  const void* v;          /* [B,H,T,S,D] */
  const float* beta;      /* [B,H,T,S] */
  const float* gamma;     /* [B,H,T] */
  const float* state_in;  /* [B,H,D,D] or NULL; seeds each direction's first frame */
  void* out;              /* [B,H,T,S,D] forward (or GDN_REVERSE) output */
  float* state_out;       /* [B,H,D,D] or NULL */
  void* out_rev;          /* GDN_BIDIR: [B,H,T,S,D] reverse-scan output */
  float* state_out_rev;   /* GDN_BIDIR: [B,H,D,D] or NULL */
  const float* w_q;       /* GDN_FUSED_PROLOGUE: [D] RMSNorm weight of q */
  const float* w_k;       /* GDN_FUSED_PROLOGUE: [D] RMSNorm weight of k */
  int B, H, T, S, D;
  int grid_h, grid_w;     /* GDN_FUSED_PROLOGUE: latent grid, grid_h*grid_w == S */
  float eps;              /* RMSNorm epsilon (0 means 1e-6) */
  float rope_base;        /* RoPE base (0 means 10000) */
  unsigned flags;
  void* workspace;        /* device scratch, 256-byte aligned */
  size_t workspace_bytes; /* >= gdn_workspace_bytes(B,H,T,S,D,flags) */
  const float* state_in_rev; /* GDN_BIDIR | GDN_REV_STATE_IN: [B,H,D,D] or NULL (zeros);
                                the chunk-causal streaming step passes the carried
                                forward state in state_in and no reverse state */
  const float* ucpe_q;    /* GDN_UCPE: [B,T,S,4,4] per-token camera matrix of q (D^T) */
  const float* ucpe_k;    /* GDN_UCPE: [B,T,S,4,4] per-token camera matrix of k (D^-1) */
} gdn_params;

/*
 * gdn_frame_scan_fwd_ex — the scan with the options of gdn_params.
 * With GDN_BIDIR the forward scan (never reset) writes out/state_out and the
 * reverse-time scan writes out_rev/state_out_rev; GDN_BLOCK_RESET then applies
 * to the reverse scan only (the chunk-causal variant of the hyper.ai summary,
 * "方法"); A_t and U_t are computed once and shared by both directions.
 * state_in seeds both directions unless GDN_REV_STATE_IN gives the reverse its
 * own (state_in_rev). Chunk-causal streaming runs one block of frames per call
 * (T = block): state_in = the previous call's state_out, GDN_REV_STATE_IN with
 * state_in_rev = NULL, so each call's reverse scan stays inside its block.
 * Returns GDN_OK or a negative status (GDN_ERR_WORKSPACE if scratch is short).
 */
GDN_API int gdn_frame_scan_fwd_ex(const gdn_params* p, gdn_stream_t stream);

/*
 * gdn_frame_scan_fwd_static — gdn_frame_scan_fwd for callers that cannot
 * allocate device memory at call time. (The pages have no counterpart: this
 * is a deployment entry point.) Streaming loops that run one short block of
 * frames per call, hosts whose device memory is all held by their own pooling
 * allocator, and plugin contexts that get no workspace pointer all fall in
 * this group: cudaMalloc / cudaFree can synchronise the device, can fail
 * while a pool owns the memory, or may be forbidden outright.
 *
 * Same arguments, results and flags as gdn_frame_scan_fwd (GDN_FUSED_PROLOGUE
 * and GDN_BIDIR are rejected). Scratch is a fixed 32 MiB array in device
 * memory inside the library, held on every GPU that loads it until the process
 * exits; nothing is allocated or freed. Sizes whose gdn_workspace_bytes exceeds
 * 32 MiB (e.g. one 3-frame block of 16 heads at 720p needs about 13 MB; a full
 * 121-frame rollout does not fit) return GDN_ERR_WORKSPACE before any launch.
 * The first call on each device looks up the array's device address (a
 * one-time runtime query); make that first call before any stream capture.
 * The address is kept for the life of the process: do not use this entry
 * point across a cudaDeviceReset, after which the array may move.
 * All calls share the array: calls ordered on one stream are safe, calls that
 * overlap on the GPU (other streams, unordered host threads) race. No part of
 * the scratch has to start at zero: a call writes every byte it reads.
 */
GDN_API int gdn_frame_scan_fwd_static(const void* q, const void* k, const void* v,
                                      const float* beta, const float* gamma,
                                      const float* state_in, void* out, float* state_out, int B,
                                      int H, int T, int S, int D, unsigned flags,
                                      gdn_stream_t stream);

/*
 * gdn_frame_scan_fwd_host — gdn_frame_scan_fwd over buffers in HOST memory
 * (the end-to-end form: inputs start and results end in host memory). Same
 * arguments, layouts, flags and results as gdn_frame_scan_fwd, except that
 * q, k, v, beta, gamma, state_in, out and state_out are host pointers
 * (page-locked memory lets the copies overlap; pageable memory works, with
 * the copies serialised). Heads are independent: the call streams them
 * through the GPU in chunks of heads_per_chunk whole heads (0: 2), with two
 * device slots alternating, so that while one chunk is scanned the next is
 * copied in and the previous copied out, on three internal streams (one
 * cudaMemcpyAsync per tensor and chunk). Device memory (two slots of inputs,
 * outputs and scan workspace for one chunk each) is taken stream-ordered from
 * `stream`'s memory pool and given back before returning. The work starts
 * after the work already enqueued on `stream`; the call returns once the
 * results are in host memory (it synchronises). Returns GDN_OK or a status.
 */
GDN_API int gdn_frame_scan_fwd_host(const void* q, const void* k, const void* v,
                                    const float* beta, const float* gamma,
                                    const float* state_in, void* out, float* state_out, int B,
                                    int H, int T, int S, int D, unsigned flags,
                                    int heads_per_chunk, gdn_stream_t stream);

/*
 * gdn_frame_scan_bwd — gradients of a loss through gdn_frame_scan_fwd.
 * (The pages print no backward; this is the adjoint of the same recurrence,
 * derived by reverse-mode differentiation.) Given dL/dO and optionally
 * dL/d(state_out), it returns dL/dq, dL/dk, dL/dv, dL/dbeta, dL/dgamma and
 * optionally dL/d(state_in) for the scan the same flags describe:
 *   G_j  = dO^T Q + gamma' (G' - G' A')       (G' of the next frame in scan
 *          order, cut where the forward scan reset the state; the last frame
 *          adds dL/d(state_out))
 *   dq   = dO S_t,  dM = S'^T G (S': the state entering the frame),
 *   dA   = -gamma dM,  dgamma = <dM, I - A>,  dU = G,
 *   dk   = beta (K^ (dA + dA^T) + V G) / sqrt(D S),  dv = beta K^ G^T,
 *   dbeta_s = k^_s . (K^ (dA + dA^T) / 2 + V G)_s.
 * Forward quantities (A_t, U_t, the states) are recomputed inside the call,
 * unless saved_workspace is set (tensor-core path: bf16, D = 128): then it
 * must be the workspace of a gdn_frame_scan_fwd_ex call with
 * GDN_SAVE_FOR_BACKWARD on the same q, k, v, beta, gamma, state_in, sizes,
 * GDN_REVERSE / GDN_BLOCK_RESET / block length, without GDN_BIDIR,
 * GDN_FUSED_PROLOGUE or GDN_FUSED_REPLAY, left untouched
 * since; the backward reads that call's A_t images and states from it and
 * skips the recompute (the saved-for-backward pattern of training). Nothing
 * can check this contract: a stale or foreign workspace gives wrong gradients.
 * Layouts and dtypes as gdn_frame_scan_fwd: d_out, dq, dk, dv like q;
 * dbeta like beta; dgamma like gamma; d_state_out, d_state_in [B,H,D,D] fp32
 * (either may be NULL). Flags: GDN_BF16, GDN_REVERSE, GDN_BLOCK_RESET,
 * GDN_MAKE_BLOCK(n), GDN_KEYS_SCALED; others return GDN_ERR_INVALID.
 * Scratch: the caller's workspace of gdn_bwd_workspace_bytes (256-byte
 * aligned). Returns GDN_OK or a negative status.
 */
typedef struct gdn_bwd_params {
  const void* q;            /* [B,H,T,S,D] */
  const void* k;            /* [B,H,T,S,D] */
  const void* v;            /* [B,H,T,S,D] */
  const float* beta;        /* [B,H,T,S] */
  const float* gamma;       /* [B,H,T] */
  const float* state_in;    /* [B,H,D,D] or NULL (zeros) */
  const void* d_out;        /* [B,H,T,S,D] dL/dO */
  const float* d_state_out; /* [B,H,D,D] dL/d(state_out) or NULL (zero) */
  void* dq;                 /* [B,H,T,S,D] */
  void* dk;                 /* [B,H,T,S,D] */
  void* dv;                 /* [B,H,T,S,D] */
  float* dbeta;             /* [B,H,T,S] */
  float* dgamma;            /* [B,H,T] */
  float* d_state_in;        /* [B,H,D,D] or NULL (not written) */
  int B, H, T, S, D;
  unsigned flags;
  void* workspace;          /* device scratch, 256-byte aligned */
  size_t workspace_bytes;   /* >= gdn_bwd_workspace_bytes(B,H,T,S,D,flags) */
  const void* saved_workspace; /* NULL, or the forward call's workspace (see above) */
} gdn_bwd_params;

GDN_API int gdn_frame_scan_bwd(const gdn_bwd_params* p, gdn_stream_t stream);
GDN_API size_t gdn_bwd_workspace_bytes(int B, int H, int T, int S, int D, unsigned flags);

/* Bytes of scratch gdn_frame_scan_fwd_ex needs for these sizes and flags
 * (0 on invalid sizes). */
GDN_API size_t gdn_workspace_bytes(int B, int H, int T, int S, int D, unsigned flags);

/*
 * gdn_frame_contract — step a2 alone: for every frame-head n in [0, N),
 *   A[n] = K^_n^T diag(beta_n) K^_n,  U[n] = V_n^T diag(beta_n) K^_n
 * with K^ = k / sqrt(D*S) (or k as given under GDN_KEYS_SCALED).
 *   k, v   [N,S,D] bf16/fp32;  beta [N,S] fp32;  A, U [N,D,D] fp32 row-major
 * Honours GDN_BF16, GDN_KEYS_SCALED, GDN_FORCE_SIMT. Returns a status.
 */
GDN_API int gdn_frame_contract(const void* k, const void* v, const float* beta, float* A, float* U,
                       int N, int S, int D, unsigned flags, gdn_stream_t stream);

/*
 * gdn_chunk_composites — step a3 alone: for each span n of L consecutive
 * frames (in the order given) with inputs A, U [n*L + j] and gamma[n*L + j],
 * j < L, the span's affine map S_start -> S_start C_n + H_n in the form
 *   C_n = g_n (I - E_n),  g_n = prod_j gamma_j
 * (E_n and H_n start at 0; each frame does E <- E + A - E A and
 *  H <- gamma (H - H A) + U). Writes E [n,D,D], H [n,D,D], g [n] fp32.
 *   A, U  [N*L,D,D] fp32;  gamma [N*L] fp32
 * Honours GDN_FORCE_SIMT. Returns a status.
 */
GDN_API int gdn_chunk_composites(const float* A, const float* U, const float* gamma, float* E, float* Hc,
                         float* g, int N, int L, int D, unsigned flags, gdn_stream_t stream);

/*
 * Time-sharded context parallelism (SANA-WM blog, Context-Parallel section:
 * each device holds a span of frames; the span's affine map
 * S_end = S_start C_p + H_p is exact, so after exchanging the maps every
 * device knows its exact start state). With R ranks holding consecutive
 * frame ranges of the same heads (rank order = time order):
 *   1. gdn_cp_shard_composite on each rank's frames -> E, H, g per head
 *      (C = g (I - E));
 *   2. all-gather E, H, g over the ranks (the caller's collective, e.g.
 *      NCCL): shard-major [R][B*H][D][D], [R][B*H];
 *   3. gdn_cp_prefix -> this rank's start state;
 *   4. gdn_frame_scan_fwd(_ex) on the rank's frames with state_in = that
 *      state; the last rank's state_out is the sequence's.
 * Forward scan order without block resets.
 *
 * gdn_cp_shard_composite: k, v [B,H,T,S,D] (dtype per GDN_BF16), beta
 * [B,H,T,S], gamma [B,H,T] of this rank's T frames; writes E, H [B,H,D,D]
 * and g [B,H] (fp32). Scratch: workspace of gdn_workspace_bytes(B,H,T,S,D,
 * flags). Flags: GDN_BF16, GDN_KEYS_SCALED, GDN_FORCE_SIMT. Returns a status.
 */
GDN_API int gdn_cp_shard_composite(const void* k, const void* v, const float* beta,
                                   const float* gamma, float* E, float* H, float* g, int B,
                                   int Hh, int T, int S, int D, unsigned flags, void* workspace,
                                   size_t workspace_bytes, gdn_stream_t stream);

/* gdn_cp_prefix: S_start of rank r = state_in (NULL = zeros) folded through
 * the maps of ranks 0..r-1: S <- g (S - S E) + H. E_all, H_all
 * [R][heads][D][D], g_all [R][heads] fp32 (shard-major, as gathered);
 * state_in, S_start [heads][D][D] fp32. Returns a status. */
GDN_API int gdn_cp_prefix(const float* E_all, const float* H_all, const float* g_all,
                          const float* state_in, float* S_start, int R, int r, int heads, int D,
                          gdn_stream_t stream);

/* Synchronises `stream`, then reads and clears the library's device status
 * word: GDN_OK, GDN_ERR_TIMEOUT if a kernel's bounded wait expired since the
 * last check, or GDN_ERR_CUDA if the stream reports an error. */
GDN_API int gdn_check_device_status(gdn_stream_t stream);

/* gdn_selftest_wait — exercises the device-side failure path without any
 * fault: one block waits on an mbarrier that is completed only when `arrive`
 * is non-zero, bounded by limit_ns nanoseconds (at most 1e9). When the wait
 * runs out the kernel records the timeout in the library's status word and
 * returns normally, so the next gdn_check_device_status reports
 * GDN_ERR_TIMEOUT and the context stays usable. Returns the launch status. */
GDN_API int gdn_selftest_wait(int arrive, long long limit_ns, gdn_stream_t stream);

/* gdn_rope_eval — the (cos, sin) pairs the fused prologue's 2-D RoPE uses,
 * for tests of their accuracy: for pair i < D/4 of an axis half and position
 * pos < npos, writes (cos, sin) of pos * rope_base^(-2i/(D/2)) to
 * cs[2 * (i * npos + pos)], cs[2 * (i * npos + pos) + 1] (device, fp32,
 * 16-byte aligned, 2 * npos * D/4 floats). reduced = 1: the angle reduced to
 * [-pi, pi] by Cody-Waite reduction, then the hardware sine/cosine, as every
 * fused-prologue kernel computes them (the contraction and the one-direction
 * readout into a shared table at start-up, the bidirectional readout per
 * token); reduced = 0: the full-precision sine/cosine of the same fp32 angle,
 * for comparison. npos in [1, 2^20].
 * Returns a status. */
GDN_API int gdn_rope_eval(int npos, int D, float rope_base, int reduced, float* cs,
                          gdn_stream_t stream);

/* Static description of a status code. */
GDN_API const char* gdn_status_string(int status);

/* One-line description of the last failure on this host thread ("" if none). */
GDN_API const char* gdn_last_error(void);

/* gdn_fault_inject — host-side fault injection for tests of the callers'
 * error paths, with no device fault: the next n calls of gdn_frame_scan_fwd,
 * gdn_frame_scan_fwd_ex, gdn_frame_scan_fwd_static and gdn_frame_scan_bwd on
 * this host thread return GDN_ERR_CUDA ("injected launch failure") once their
 * arguments have passed the checks, before anything is launched (the plain
 * entry has already taken its stream-ordered workspace, which it frees).
 * Outputs are left untouched. n <= 0 disarms. Returns the number of injected
 * failures still pending before this call. */
GDN_API int gdn_fault_inject(int n);

/* Kernel launches made by this host thread's gdn_* calls since the last reset;
 * reset = 1 clears the counter after reading it. */
GDN_API long long gdn_launch_count(int reset);

/* Phase timing: while enabled, every kernel the library launches from this
 * host thread is bracketed by two CUDA events recorded on its launch stream
 * (instrumentation for benchmarks; no host synchronisation). enable = 1
 * starts a fresh record, enable = 0 stops recording. Returns GDN_OK. */
GDN_API int gdn_profile_enable(int enable);

/* Sums the recorded kernel durations per phase, waiting on the events:
 * ms[i] and counts[i] for phase i < n, with phases 0 prologue, 1 contract,
 * 2 compose, 3 prefix, 4 scan/replay, 5 readout, 6 replay fused with the
 * readout, 7 contraction with the sequential scan alongside; backward:
 * 8 recompute, 9 dO^T Q, 10 adjoint chain, 11 per-frame terms, 12 token
 * gradients, 13 dq. Returns the number of phases written, or a negative
 * status. */
GDN_API int gdn_profile_read(double* ms, long long* counts, int n);

/* ABI version: major * 10000 + minor * 100 + patch. */
GDN_API int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
