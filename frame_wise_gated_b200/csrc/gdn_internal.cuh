// Internal declarations shared by the kernels and the C ABI of libgdnscan.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

// ---- scalar load/store by element type -------------------------------------
template <typename T>
__device__ __forceinline__ float ldf(const T* p);
template <>
__device__ __forceinline__ float ldf<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ void stf(T* p, float x);
template <>
__device__ __forceinline__ void stf<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void stf<__nv_bfloat16>(__nv_bfloat16* p, float x) {
  *p = __float2bfloat16_rn(x);
}

// ---- scan plan ---------------------------------------------------------------
// How the frames of one direction are cut into chains of the recurrence.
enum SegMode : int {
  SEG_SEQUENTIAL = 0,  // one chain over all T frames (block resets inside it)
  SEG_CHUNKS = 1,      // uniform spans of L frames in scan order, composed
  SEG_BLOCKS = 2,      // one chain per reset block (blocks are independent)
};

enum ChainMode : int {
  CHAIN_SCAN = 0,     // S <- gamma (S - S A) + U per frame, store S_t
  CHAIN_COMPOSE = 1,  // per span: E <- E + A - E A and H <- gamma (H - H A) + U
  CHAIN_PREFIX = 2,   // per head: S_start(p+1) = g_p (S_start(p) - S_start(p) E_p) + H_p
  CHAIN_ADJOINT = 3,  // backward: per head, G_j = W_j + g_{j+1} (G_{j+1} - G_{j+1} A_{j+1})
};

// Everything the chain kernels need; pointers are device pointers.
struct ChainArgs {
  int mode;       // ChainMode
  int seg;        // SegMode
  int D, T;
  int L;          // chunk length (SEG_CHUNKS)
  int block;      // reset block length (SEG_BLOCKS, or resets inside SEG_SEQUENTIAL)
  int seq_reset;  // SEG_SEQUENTIAL: zero the state on entering a new block
  int reverse;
  int nseg;       // chains per head: 1, ceil(T/L) or ceil(T/block)
  int heads;      // B*H
  const float* A;         // [heads*T, D, D]
  const float* U;         // [heads*T, D, D]
  const float* gamma;     // [heads*T]
  const float* state_in;  // [heads, D, D] or null
  float* state_out;       // [heads, D, D] or null
  float* Sfr;             // per-frame states [heads*T, D, D] fp32, or bf16 hi/lo pairs
  int sfr_hilo;           // 1: Sfr holds [heads*T][2][D][D] bf16 (hi, lo)
  float* E;               // [heads*nseg, D, D]
  float* Hc;              // [heads*nseg, D, D]
  float* g;               // [heads*nseg]
  float* Sst;             // [heads*nseg, D, D] span start states
  int y_image;            // A (and E for the prefix) are stored as bf16 operand images
  int e_image;            // the compose chain writes E as an operand image
  int sst_hilo;           // Sst holds [heads*nseg][2][D][D] bf16 (hi, lo) pairs
  // backward (CHAIN_ADJOINT)
  const float* Zw;        // [heads*T, D, D] W_t = dO_t^T Q_t
  float* Gout;            // [heads*T, D, D] total state gradients G_t
  const float* dS_out;    // [heads, D, D] gradient of state_out, or null
  float* dS_in;           // [heads, D, D] gradient of state_in, or null
  const void* zero_img;   // an all-zero operand image (tensor-core adjoint chain)
};

// An "operand image" of a D x D fp32 matrix M (D = 128) is the exact
// shared-memory tile the tensor-core chain kernel uses as its B operand
// B[k][n] = M[k][n]: a bf16 (hi, lo) pair, hi = bf16(M), lo = bf16(M - hi),
// each as two 64-column blocks of 128 rows x 128 bytes in the 128-byte
// swizzled MN-major layout (hi: bytes [0, 32K), lo: [32K, 64K)). It occupies
// the same 64 KiB as the fp32 matrix and is copied into shared memory with a
// single bulk copy.
constexpr int kImageBytes = 128 * 128 * 4;

// Scan-order helpers (host and device).
__host__ __device__ __forceinline__ int frame_at(int j, int T, int reverse) {
  return reverse ? T - 1 - j : j;
}
// Range [j0, j1) of scan positions covered by chain p.
__host__ __device__ __forceinline__ void seg_range(const ChainArgs& a, int p, int* j0, int* j1) {
  if (a.seg == SEG_SEQUENTIAL) {
    *j0 = 0;
    *j1 = a.T;
  } else if (a.seg == SEG_CHUNKS) {
    *j0 = p * a.L;
    *j1 = min(*j0 + a.L, a.T);
  } else {
    int nb = (a.T + a.block - 1) / a.block;
    int blk = a.reverse ? nb - 1 - p : p;
    int t0 = blk * a.block, t1 = min(t0 + a.block, a.T);
    if (a.reverse) {
      *j0 = a.T - t1;
      *j1 = a.T - t0;
    } else {
      *j0 = t0;
      *j1 = t1;
    }
  }
}

// ---- workspace layout ---------------------------------------------------------
struct Layout {
  size_t A, U, Sfr, Sfr2, E, Hc, g, Sst, qh, kh, flags, total;
  int nseg_max;
};

Layout make_layout(int B, int H, int T, int S, int D, unsigned flags);

// ---- launch bookkeeping --------------------------------------------------------
void count_launch(int n = 1);

// ---- SIMT (CUDA-core) kernels: any D in {16..256}, fp32 or bf16 -----------------
// mq, mk: per-token camera matrices [B][T][S][4][4] (both null: no camera
// encoding, RoPE on all D channels); H, T locate a frame-head's (b, t).
cudaError_t simt_prologue(bool bf16, const void* q_raw, const void* k_raw, const float* w_q,
                          const float* w_k, void* q_out, void* k_out, long long frames, int S,
                          int grid_w, int D, float eps, float base, float kscale,
                          cudaStream_t st, const float* mq = nullptr, const float* mk = nullptr,
                          int H = 1, int T = 1);
cudaError_t simt_contract(bool bf16, const void* k, const void* v, const float* beta, float* A,
                          float* U, long long N, int S, int D, float cA, float cU,
                          cudaStream_t st);
cudaError_t simt_chain(const ChainArgs& a, int nchains, cudaStream_t st);
// Context parallelism: start state of shard r from shard-major maps (E, H, g).
cudaError_t simt_cp_prefix(const float* E, const float* Hc, const float* g, const float* s0,
                           float* out, int r, int heads, int D, cudaStream_t st);
cudaError_t simt_readout(bool bf16, const void* q, const float* Sfr, void* out, long long N,
                         int S, int D, cudaStream_t st);

// ---- backward (CUDA cores) ------------------------------------------------------
// dM_j = S'_j^T G_j per frame (S'_j: state entering frame j of the scan order).
// hilo: Sfr and G hold bf16 (hi, lo) pairs [F][2][D][D] instead of fp32.
cudaError_t simt_bwd_dm(const void* Sfr, const float* state_in, const void* G, float* dM,
                        long long N, int T, int D, int reverse, int seq_reset, int block,
                        bool hilo, cudaStream_t st);
// In place dM -> dA + dA^T = -gamma (dM + dM^T); dgamma = <dM, I - A>. A is
// fp32 or (a_image, D = 128) operand images; with bimg (D = 128, G_hilo set)
// also writes the tensor-core token kernel's per-frame B operand (64 KiB).
cudaError_t simt_bwd_dterm(float* dM, const void* A, bool a_image, const float* gamma,
                           float* dgamma, long long N, int D, const void* G_hilo, void* bimg,
                           cudaStream_t st);
// dL/d(state_in) = g (G - G A) at the first frame t0 of each head (D = 128,
// G as (hi, lo) pairs, A as operand images).
cudaError_t simt_bwd_ds0(const void* G_hilo, const void* A_img, const float* gamma, float* ds0,
                         int heads, int T, int t0, cudaStream_t st);
// Per frame n: out[s, :] = scale * x[s, :] M_n^T (trans = 0) or x[s, :] M_n (trans = 1).
cudaError_t simt_rowmat(bool bf16_in, bool f32_out, int trans, const void* x, const float* M,
                        void* out, long long N, int S, int D, float scale, cudaStream_t st);
// dk, dv, dbeta per token from the products P2, P3, P5.
cudaError_t simt_bwd_combine(bool bf16, const void* k, const float* beta, const float* P2,
                             const float* P3, const float* P5, void* dk, void* dv, float* dbeta,
                             long long ntok, int D, float c, cudaStream_t st);

// ---- tensor-core (tcgen05) kernels, bf16, sm_100a -------------------------------
// Prologue applied inside the tensor-core loaders (RMSNorm -> ReLU -> 2-D RoPE;
// the key scale is folded into the contraction's epilogue constants).
struct ProArgs {
  const float* w;    // [D] RMSNorm weight
  int grid_w;
  float eps;
  int npos;
  float base;        // RoPE base (pair i turns by pos * base^(-2i/(D/2)))
  const float* ucpe; // null, or this side's camera matrices [B][T][S][4][4]: channels
                     // [0, D/2) in blocks of 4 take them, the RoPE takes [D/2, D)
  int H, T;          // heads and frames: frame-head n = (b * H + h) * T + t
};
// (cos, sin) table, pair-major: cs[i * npos + pos], pos < npos, i < D/4
// (consecutive tokens of a row read consecutive entries).
cudaError_t rope_table(float2* cs, int npos, int D, float base, cudaStream_t st);
cudaError_t rope_reduced(float2* cs, int npos, int D, float base, cudaStream_t st);

// Largest max(grid_h, grid_w) the fused prologue's shared-memory table holds (D = 128).
int tc_prologue_max_positions();
bool tc_contract_supported(int D);
cudaError_t tc_contract(const void* k, const void* v, const float* beta, float* A, float* U,
                        long long N, int S, int D, float cA, float cU, int a_image,
                        const ProArgs* pro, cudaStream_t st);
// Token-split contraction (D = 128): `parts` CTAs per frame-head add partial
// A_t, U_t into fp32 Aacc, U (both zeroed here); Aacc still needs tc_to_image.
cudaError_t tc_contract_split(const void* k, const void* v, const float* beta, float* Aacc,
                              float* U, long long N, int S, float cA, float cU, int parts,
                              const ProArgs* pro, cudaStream_t st);
// fp32 D x D matrices -> operand images (D = 64 or 128).
cudaError_t tc_to_image(const float* src, void* dst, long long n, int D, cudaStream_t st);
bool tc_readout_supported(int D);
cudaError_t tc_readout(const void* q, const void* Sfr_hilo, void* out, long long N, int S, int D,
                       const ProArgs* pro, cudaStream_t st);
// Replay of CHAIN_SCAN chains fused with the readout (bf16 out, no prologue).
bool tc_scan_readout_supported(int D);
cudaError_t tc_scan_readout(const ChainArgs& a, int nchains, const void* q, void* out, int S,
                            cudaStream_t st);
// Both directions' readouts in one pass over Q (bf16 out, D = 128).
bool tc_readout2_supported(int D);
cudaError_t tc_readout2(const void* q, const void* sfr_f, const void* sfr_r, void* out_f,
                        void* out_r, long long N, int S, int D, const ProArgs* pro,
                        cudaStream_t st);
// ---- contraction with the sequential scan alongside (one cooperative launch) ----
// One direction of the overlapped scan.
struct OvlDir {
  int reverse;     // scan order T-1 .. 0
  int blocks_asc;  // reverse scan reset per block, run block by block in
                   // ascending time (frames descending inside each block)
  int seq_reset;   // zero the state on entering a new block in scan order
  const float* state_in;  // [heads, D, D] or null (adjoint: dL/d(state_out))
  float* state_out;       // [heads, D, D] or null
  int adjoint;     // backward: G over the forward scan (direction `reverse`)
                   // backwards, G <- W_t + g' (G - G A') with A' = A of the
                   // next forward frame (from `A`); the launch's contraction
                   // computes W_t into its U output
};

struct OvlArgs {
  int heads, T, block, ndir;
  const float* gamma;
  const uint8_t* A;  // operand images of A_t, [heads*T][kImageBytes]
  int* flags;        // [heads*T], zero before the launch
  OvlDir dir[2];
  const uint8_t* zero_img;  // adjoint: an all-zero operand image
  int a_image;       // the contraction's A output: 1 operand images, 2 not written
  int contract_rev;  // the contraction visits frames in reverse time
  const float* U;    // U_t [heads*T][D][D] (set by tc_contract_scan)
  int discard;       // one direction only: once a chain has copied a frame's operands
                     // their L2 lines are dropped unwritten: 1 = U_t, 2 = the A_t image
};

bool tc_overlap_supported(int D);
int tc_num_sms();
// Most chains one overlapped launch runs (the rest of the SMs contract).
int tc_overlap_max_chains();
// Contraction of all frame-heads (A_t as operand images, U_t fp32) while
// o.ndir * o.heads CTAs run the sequential chains, storing each frame's state
// as a bf16 (hi, lo) pair into sfr0 (direction 0) / sfr1 (direction 1).
cudaError_t tc_contract_scan(const void* k, const void* v, const float* beta, float* A, float* U,
                             long long N, int S, float cA, float cU, const ProArgs* pro,
                             const OvlArgs& o, void* sfr0, void* sfr1, cudaStream_t st);
// Backward, D = 128: dq = dO S_t (S_t as hi/lo pairs) and the token gradients
// dk, dv, dbeta from the per-frame B operand [dA + dA^T ; G] (64 KiB bf16).
cudaError_t tc_readout_trans(const void* x, const void* Sfr_hilo, void* out, long long N, int S,
                             cudaStream_t st);
// Per-frame backward terms on tensor cores: dA + dA^T and G into the token
// kernel's operand, dgamma. s0_hilo: scratch for state_in as hi/lo pairs
// (heads x 64 KiB); zero_hilo: 64 KiB of zeros.
cudaError_t tc_bwd_frames(const void* Sfr_hilo, const float* state_in, void* s0_hilo,
                          const void* zero_hilo, const void* G_hilo, const void* A_img,
                          const float* gamma, float* dgamma, void* bimg, long long N, int heads,
                          int T, int reverse, int seq_reset, int block, cudaStream_t st);
cudaError_t tc_bwd_tokens(const void* k, const void* v, const float* beta, const void* bimg,
                          void* dk, void* dv, float* dbeta, long long N, int S, float c,
                          cudaStream_t st);
bool tc_chain_supported(int D);
cudaError_t tc_chain(const ChainArgs& a, int nchains, cudaStream_t st);
cudaError_t tc_selftest_wait(int arrive, long long limit_ns, cudaStream_t st);
// Reads and clears the device status word of the tensor-core kernels.
cudaError_t tc_read_status(int* status, cudaStream_t st);

}  // namespace gdn
