// CUDA-core (SIMT) kernels of the frame-wise GDN scan.
//
// These carry the fp32 dtype path, every head dimension D in {16, ..., 256},
// and serve as the in-library cross-check of the tensor-core kernels. All
// arithmetic is fp32 with fp32 accumulation.
//
// Recurrence (SANA-WM blog, blog.hotdry.top, section 混合线性注意力):
//   A_t = K^^T diag(beta) K^,  U_t = V^T diag(beta) K^,  K^ = K / sqrt(D*S)
//   S_t = gamma_t (S_{t-1} - S_{t-1} A_t) + U_t,  O_t = Q_t S_t^T.
// Span composition (same page, Context-Parallel section): S_end = S_start C + H.
#include "gdn_internal.cuh"

namespace gdn {

// ----------------------------------------------------------------------------
// Prologue: RMSNorm -> ReLU -> key scale -> 2-D spatial RoPE, one warp per token
// (SANA-WM blog, Context-Parallel section, the fused-op order). With UCPE the
// camera encoding (same page, section 双分支相机控制) takes channels [0, D/2):
// each block of 4 channels of token (b, t, s) is multiplied by that token's
// 4 x 4 matrix (mq for queries, mk for keys: [B][T][S][4][4] fp32, shared by
// the heads), and the RoPE acts on [D/2, D) as a vector of D/2 channels.
// ----------------------------------------------------------------------------
template <typename T, bool UCPE>
__global__ void __launch_bounds__(256)
    k_prologue(const T* __restrict__ qin, const T* __restrict__ kin, const float* __restrict__ wq,
               const float* __restrict__ wk, T* __restrict__ qout, T* __restrict__ kout,
               long long ntok, int S, int grid_w, int D, float eps, float base, float kscale,
               const float* __restrict__ mq, const float* __restrict__ mk, int H, int Tn) {
  const long long tok = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tok >= ntok) return;  // warp-uniform: one token per warp
  const int which = blockIdx.y;  // 0: q, 1: k
  const T* in = which ? kin : qin;
  T* out = which ? kout : qout;
  const float* w = which ? wk : wq;
  const float scale = which ? kscale : 1.0f;
  const size_t off = (size_t)tok * D;
  const int s = (int)(tok % S);
  const int py = s / grid_w, px = s % grid_w;
  const int npairs = D >> 1;
  // RoPE channels: all D (pairs from 0), or the upper D/2 with UCPE
  const int rope_p0 = UCPE ? D >> 2 : 0, rope_ch = UCPE ? D >> 1 : D;
  const int quarter = rope_ch >> 2, half = rope_ch >> 1;

  float a[4], b[4];
  float ss = 0.f;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int p = lane + 32 * m;
    a[m] = b[m] = 0.f;
    if (p < npairs) {
      a[m] = ldf(in + off + 2 * p);
      b[m] = ldf(in + off + 2 * p + 1);
      ss += a[m] * a[m] + b[m] * b[m];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss / (float)D + eps);
  float M[16];
  if (UCPE) {
    const long long n = tok / S;  // frame-head (b * H + h) * T + t
    const long long bt = (n / ((long long)H * Tn)) * Tn + n % Tn;
    const float4* src = (const float4*)((which ? mk : mq) + ((size_t)bt * S + s) * 16);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float4 v = __ldg(src + r);
      M[4 * r] = v.x; M[4 * r + 1] = v.y; M[4 * r + 2] = v.z; M[4 * r + 3] = v.w;
    }
  }
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int p = lane + 32 * m;
    // every lane of a warp takes the same m-iterations, so the shuffle below
    // sees all 32 lanes (pairs past D/2 simply hold zeros)
    const float x0 = p < npairs ? fmaxf(a[m] * inv * w[2 * p], 0.f) * scale : 0.f;
    const float x1 = p < npairs ? fmaxf(b[m] * inv * w[2 * p + 1], 0.f) * scale : 0.f;
    if (UCPE && 32 * m < rope_p0) {
      // camera block p / 2: this lane's pair and its neighbour's (lane ^ 1)
      const float y0 = __shfl_xor_sync(0xffffffffu, x0, 1);
      const float y1 = __shfl_xor_sync(0xffffffffu, x1, 1);
      if (p < rope_p0) {
        const int hi = p & 1;  // rows 2, 3 of the block for the odd pair
        const float v0 = hi ? y0 : x0, v1 = hi ? y1 : x1, v2 = hi ? x0 : y0, v3 = hi ? x1 : y1;
        const float* r0 = M + 8 * hi;
        stf(out + off + 2 * p, r0[0] * v0 + r0[1] * v1 + r0[2] * v2 + r0[3] * v3);
        stf(out + off + 2 * p + 1, r0[4] * v0 + r0[5] * v1 + r0[6] * v2 + r0[7] * v3);
        continue;
      }
    }
    if (p < npairs) {
      const int pr = p - rope_p0;  // pair index inside the RoPE channels
      const int hsel = pr / quarter, i = pr % quarter;
      const float pos = hsel ? (float)px : (float)py;
      const float theta = powf(base, -2.0f * (float)i / (float)half);
      float sn, cs;
      sincosf(pos * theta, &sn, &cs);
      stf(out + off + 2 * p, x0 * cs - x1 * sn);
      stf(out + off + 2 * p + 1, x0 * sn + x1 * cs);
    }
  }
}

cudaError_t simt_prologue(bool bf16, const void* q_raw, const void* k_raw, const float* w_q,
                          const float* w_k, void* q_out, void* k_out, long long frames, int S,
                          int grid_w, int D, float eps, float base, float kscale,
                          cudaStream_t st, const float* mq, const float* mk, int H, int T) {
  const long long ntok = frames * S;
  dim3 grid((unsigned)((ntok + 7) / 8), 2);
  const bool ucpe = mq && mk;
  if (bf16 && ucpe)
    k_prologue<__nv_bfloat16, true><<<grid, 256, 0, st>>>(
        (const __nv_bfloat16*)q_raw, (const __nv_bfloat16*)k_raw, w_q, w_k,
        (__nv_bfloat16*)q_out, (__nv_bfloat16*)k_out, ntok, S, grid_w, D, eps, base, kscale, mq,
        mk, H, T);
  else if (bf16)
    k_prologue<__nv_bfloat16, false><<<grid, 256, 0, st>>>(
        (const __nv_bfloat16*)q_raw, (const __nv_bfloat16*)k_raw, w_q, w_k,
        (__nv_bfloat16*)q_out, (__nv_bfloat16*)k_out, ntok, S, grid_w, D, eps, base, kscale, mq,
        mk, H, T);
  else if (ucpe)
    k_prologue<float, true><<<grid, 256, 0, st>>>((const float*)q_raw, (const float*)k_raw, w_q,
                                                  w_k, (float*)q_out, (float*)k_out, ntok, S,
                                                  grid_w, D, eps, base, kscale, mq, mk, H, T);
  else
    k_prologue<float, false><<<grid, 256, 0, st>>>((const float*)q_raw, (const float*)k_raw, w_q,
                                                   w_k, (float*)q_out, (float*)k_out, ntok, S,
                                                   grid_w, D, eps, base, kscale, mq, mk, H, T);
  count_launch();
  return cudaGetLastError();
}

// ----------------------------------------------------------------------------
// Per-frame contraction (step a2): A = cA K^T diag(beta) K, U = cU V^T diag(beta) K.
// One CTA per (frame, TILE x TILE output tile); tokens streamed 32 at a time.
// ----------------------------------------------------------------------------
template <typename T, int TILE>
__global__ void __launch_bounds__(256)
    k_contract_simt(const T* __restrict__ k, const T* __restrict__ v,
                    const float* __restrict__ beta, float* __restrict__ A, float* __restrict__ U,
                    int S, int D, float cA, float cU) {
  constexpr int R = TILE / 16;
  constexpr int KC = 32;
  __shared__ float Ki[KC][TILE];
  __shared__ float Kj[KC][TILE];  // beta * k, columns of the tile
  __shared__ float Vi[KC][TILE];
  const long long n = blockIdx.x;
  const int nt = D / TILE;
  const int ti = blockIdx.y / nt, tj = blockIdx.y % nt;
  const T* kf = k + (size_t)n * S * D;
  const T* vf = v + (size_t)n * S * D;
  const float* bf = beta ? beta + (size_t)n * S : nullptr;  // null: beta = 1
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float accA[R][R], accU[R][R];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int j = 0; j < R; ++j) accA[i][j] = accU[i][j] = 0.f;

  for (int s0 = 0; s0 < S; s0 += KC) {
    for (int e = threadIdx.x; e < KC * TILE; e += 256) {
      const int r = e / TILE, c = e % TILE, s = s0 + r;
      float ki = 0.f, kj = 0.f, vi = 0.f;
      if (s < S) {
        ki = ldf(kf + (size_t)s * D + ti * TILE + c);
        kj = ldf(kf + (size_t)s * D + tj * TILE + c) * (bf ? bf[s] : 1.0f);
        vi = ldf(vf + (size_t)s * D + ti * TILE + c);
      }
      Ki[r][c] = ki;
      Kj[r][c] = kj;
      Vi[r][c] = vi;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < KC; ++r) {
      float a[R], vv[R], bb[R];
#pragma unroll
      for (int i = 0; i < R; ++i) {
        a[i] = Ki[r][ty * R + i];
        vv[i] = Vi[r][ty * R + i];
        bb[i] = Kj[r][tx * R + i];
      }
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < R; ++j) {
          accA[i][j] = fmaf(a[i], bb[j], accA[i][j]);
          accU[i][j] = fmaf(vv[i], bb[j], accU[i][j]);
        }
    }
    __syncthreads();
  }
  float* An = A ? A + (size_t)n * D * D : nullptr;
  float* Un = U + (size_t)n * D * D;
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const size_t idx = (size_t)(ti * TILE + ty * R + i) * D + tj * TILE + tx * R + j;
      if (A) An[idx] = accA[i][j] * cA;  // null A: only U is wanted
      Un[idx] = accU[i][j] * cU;
    }
}

template <typename T>
static cudaError_t contract_t(const void* k, const void* v, const float* beta, float* A,
                              float* U, long long N, int S, int D, float cA, float cU,
                              cudaStream_t st) {
  const int tile = D < 64 ? D : 64;
  dim3 grid((unsigned)N, (D / tile) * (D / tile));
  switch (tile) {
    case 16:
      k_contract_simt<T, 16><<<grid, 256, 0, st>>>((const T*)k, (const T*)v, beta, A, U, S, D,
                                                   cA, cU);
      break;
    case 32:
      k_contract_simt<T, 32><<<grid, 256, 0, st>>>((const T*)k, (const T*)v, beta, A, U, S, D,
                                                   cA, cU);
      break;
    default:
      k_contract_simt<T, 64><<<grid, 256, 0, st>>>((const T*)k, (const T*)v, beta, A, U, S, D,
                                                   cA, cU);
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t simt_contract(bool bf16, const void* k, const void* v, const float* beta, float* A,
                          float* U, long long N, int S, int D, float cA, float cU,
                          cudaStream_t st) {
  return bf16 ? contract_t<__nv_bfloat16>(k, v, beta, A, U, N, S, D, cA, cU, st)
              : contract_t<float>(k, v, beta, A, U, N, S, D, cA, cU, st);
}

// ----------------------------------------------------------------------------
// Chains of the recurrence X <- alpha (X - X Y) + Z (steps a3, a4, a5).
// Each state row evolves on its own (row i of X Y needs only row i of X), so a
// CTA owns 16 rows of one chain; Y is streamed through shared memory 16 rows
// of k at a time. Thread (r, l): row r = tid / 16, columns l + 16 m.
// ----------------------------------------------------------------------------
constexpr int kChainRows = 16;

template <int D>
__device__ __forceinline__ void chain_step(float* X, float* Yc, const float* __restrict__ Y,
                                           const float* __restrict__ Z, float alpha, int row0,
                                           bool reset) {
  constexpr int NM = D / 16;
  const int r = threadIdx.x >> 4, l = threadIdx.x & 15;
  float acc[NM];
#pragma unroll
  for (int m = 0; m < NM; ++m) acc[m] = 0.f;
  for (int k0 = 0; Y && k0 < D; k0 += 16) {  // null Y: X Y = 0
    for (int e = threadIdx.x; e < 16 * D; e += 256) Yc[e] = Y[(size_t)k0 * D + e];
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < 16; ++kk) {
      const float x = X[r * D + k0 + kk];
#pragma unroll
      for (int m = 0; m < NM; ++m) acc[m] = fmaf(x, Yc[kk * D + l + 16 * m], acc[m]);
    }
    __syncthreads();
  }
  const int row = row0 + r;
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    const int c = l + 16 * m;
    const float z = Z ? Z[(size_t)row * D + c] : 0.f;
    X[r * D + c] = reset ? z : alpha * (X[r * D + c] - acc[m]) + z;
  }
  __syncthreads();
}

__device__ __forceinline__ void rows_store(const float* X, float* dst, int D, int row0) {
  const int r = threadIdx.x >> 4, l = threadIdx.x & 15;
  const int row = row0 + r;
  if (row < D)
    for (int c = l; c < D; c += 16) dst[(size_t)row * D + c] = X[r * D + c];
}

__device__ __forceinline__ void rows_store_hilo(const float* X, __nv_bfloat16* dst, int D,
                                                int row0) {
  const int r = threadIdx.x >> 4, l = threadIdx.x & 15;
  const int row = row0 + r;
  if (row < D)
    for (int c = l; c < D; c += 16) {
      const float x = X[r * D + c];
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      dst[(size_t)row * D + c] = hi;
      dst[(size_t)D * D + (size_t)row * D + c] = __float2bfloat16_rn(x - __bfloat162float(hi));
    }
}

__device__ __forceinline__ void rows_load(float* X, const float* src, int D, int row0) {
  const int r = threadIdx.x >> 4, l = threadIdx.x & 15;
  const int row = row0 + r;
  for (int c = l; c < D; c += 16) X[r * D + c] = (src && row < D) ? src[(size_t)row * D + c] : 0.f;
  __syncthreads();
}

template <int D>
__global__ void __launch_bounds__(256) k_chain_simt(ChainArgs a) {
  extern __shared__ float smem[];
  const int T = a.T;
  float* X = smem;                    // [16][D]
  float* Yc = smem + kChainRows * D;  // [16][D]
  const int row0 = blockIdx.y * kChainRows;
  const int c = blockIdx.x;

  if (a.mode == CHAIN_SCAN) {
    const int bh = c / a.nseg, p = c % a.nseg;
    int j0, j1;
    seg_range(a, p, &j0, &j1);
    const float* init = nullptr;
    if (p == 0) {
      init = a.state_in ? a.state_in + (size_t)bh * D * D : nullptr;
    } else if (a.seg == SEG_CHUNKS) {
      init = a.Sst + ((size_t)bh * a.nseg + p) * D * D;
    }
    rows_load(X, init, D, row0);
    int tprev = -1;
    for (int j = j0; j < j1; ++j) {
      const int t = frame_at(j, T, a.reverse);
      const bool rst = a.seg == SEG_SEQUENTIAL && a.seq_reset && j > 0 &&
                       (t / a.block) != (tprev / a.block);
      tprev = t;
      const size_t fi = (size_t)bh * T + t;
      chain_step<D>(X, Yc, a.A + fi * D * D, a.U + fi * D * D, a.gamma[fi], row0, rst);
      if (a.sfr_hilo)
        rows_store_hilo(X, (__nv_bfloat16*)a.Sfr + fi * 2 * D * D, D, row0);
      else
        rows_store(X, a.Sfr + fi * D * D, D, row0);
      if (j == T - 1 && a.state_out) rows_store(X, a.state_out + (size_t)bh * D * D, D, row0);
    }
  } else if (a.mode == CHAIN_COMPOSE) {
    const int half = a.heads * a.nseg;
    const int which = c >= half;  // 0: E, 1: H
    const int cc = which ? c - half : c;
    const int bh = cc / a.nseg, p = cc % a.nseg;
    int j0, j1;
    seg_range(a, p, &j0, &j1);
    rows_load(X, nullptr, D, row0);
    float gp = 1.f;
    for (int j = j0; j < j1; ++j) {
      const int t = frame_at(j, T, a.reverse);
      const size_t fi = (size_t)bh * T + t;
      const float* Af = a.A + fi * D * D;
      if (which)
        chain_step<D>(X, Yc, Af, a.U + fi * D * D, a.gamma[fi], row0, false);
      else
        chain_step<D>(X, Yc, Af, Af, 1.0f, row0, false);
      gp *= a.gamma[fi];
    }
    const size_t si = (size_t)bh * a.nseg + p;
    rows_store(X, (which ? a.Hc : a.E) + si * D * D, D, row0);
    if (!which && blockIdx.y == 0 && threadIdx.x == 0) a.g[si] = gp;
  } else if (a.mode == CHAIN_ADJOINT) {
    // Adjoint of a sequential scan (backward pass): per head, scan positions
    // j = T-1 .. 0; G_j = W_j + g_{j+1} (G_{j+1} - G_{j+1} A_{j+1}) with the
    // carry cut where the forward scan reset the state before position j+1,
    // and G_{T-1} = W_{T-1} + dL/d(state_out). Each G_j is stored; finally the
    // gradient of state_in, g_0 (G_0 - G_0 A_0).
    const int bh = c;
    rows_load(X, a.dS_out ? a.dS_out + (size_t)bh * D * D : nullptr, D, row0);
    for (int j = T - 1; j >= 0; --j) {
      const int t = frame_at(j, T, a.reverse);
      const size_t fi = (size_t)bh * T + t;
      if (j == T - 1) {
        chain_step<D>(X, Yc, nullptr, a.Zw + fi * D * D, 1.0f, row0, false);
      } else {
        const int tn = frame_at(j + 1, T, a.reverse);
        const bool cut = a.seq_reset && (t / a.block) != (tn / a.block);
        const size_t fn = (size_t)bh * T + tn;
        chain_step<D>(X, Yc, a.A + fn * D * D, a.Zw + fi * D * D, a.gamma[fn], row0, cut);
      }
      rows_store(X, a.Gout + fi * D * D, D, row0);
    }
    if (a.dS_in) {
      const size_t f0 = (size_t)bh * T + frame_at(0, T, a.reverse);
      chain_step<D>(X, Yc, a.A + f0 * D * D, nullptr, a.gamma[f0], row0, false);
      rows_store(X, a.dS_in + (size_t)bh * D * D, D, row0);
    }
  } else {  // CHAIN_PREFIX
    const int bh = c;
    rows_load(X, a.state_in ? a.state_in + (size_t)bh * D * D : nullptr, D, row0);
    for (int p = 0; p < a.nseg; ++p) {
      const size_t si = (size_t)bh * a.nseg + p;
      rows_store(X, a.Sst + si * D * D, D, row0);
      if (p + 1 < a.nseg)
        chain_step<D>(X, Yc, a.E + si * D * D, a.Hc + si * D * D, a.g[si], row0, false);
    }
  }
}

template <int D>
static cudaError_t chain_t(const ChainArgs& a, int nchains, cudaStream_t st) {
  const size_t smem = 2 * kChainRows * D * sizeof(float);
  dim3 grid((unsigned)nchains, (D + kChainRows - 1) / kChainRows);
  k_chain_simt<D><<<grid, 256, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

// Context-parallel prefix: S_start of shard r = state_in folded through the
// affine maps of shards 0..r-1 (S <- g (S - S E) + H), maps shard-major
// [R][heads][D][D]. CTA = (head, 16 rows).
template <int D>
__global__ void __launch_bounds__(256)
    k_cp_prefix(const float* __restrict__ E, const float* __restrict__ Hc,
                const float* __restrict__ g, const float* __restrict__ state_in,
                float* __restrict__ out, int r, int heads) {
  extern __shared__ float smem[];
  float* X = smem;
  float* Yc = smem + kChainRows * D;
  const int bh = blockIdx.x, row0 = blockIdx.y * kChainRows;
  rows_load(X, state_in ? state_in + (size_t)bh * D * D : nullptr, D, row0);
  for (int p = 0; p < r; ++p) {
    const size_t si = (size_t)p * heads + bh;
    chain_step<D>(X, Yc, E + si * D * D, Hc + si * D * D, g[si], row0, false);
  }
  rows_store(X, out + (size_t)bh * D * D, D, row0);
}

template <int D>
static cudaError_t cp_prefix_t(const float* E, const float* Hc, const float* g, const float* s0,
                               float* out, int r, int heads, cudaStream_t st) {
  const size_t smem = 2 * kChainRows * D * sizeof(float);
  dim3 grid((unsigned)heads, (D + kChainRows - 1) / kChainRows);
  k_cp_prefix<D><<<grid, 256, smem, st>>>(E, Hc, g, s0, out, r, heads);
  count_launch();
  return cudaGetLastError();
}

cudaError_t simt_cp_prefix(const float* E, const float* Hc, const float* g, const float* s0,
                           float* out, int r, int heads, int D, cudaStream_t st) {
  switch (D) {
    case 16: return cp_prefix_t<16>(E, Hc, g, s0, out, r, heads, st);
    case 32: return cp_prefix_t<32>(E, Hc, g, s0, out, r, heads, st);
    case 64: return cp_prefix_t<64>(E, Hc, g, s0, out, r, heads, st);
    case 128: return cp_prefix_t<128>(E, Hc, g, s0, out, r, heads, st);
    case 256: return cp_prefix_t<256>(E, Hc, g, s0, out, r, heads, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t simt_chain(const ChainArgs& a, int nchains, cudaStream_t st) {
  switch (a.D) {
    case 16: return chain_t<16>(a, nchains, st);
    case 32: return chain_t<32>(a, nchains, st);
    case 64: return chain_t<64>(a, nchains, st);
    case 128: return chain_t<128>(a, nchains, st);
    case 256: return chain_t<256>(a, nchains, st);
    default: return cudaErrorInvalidValue;
  }
}

// ----------------------------------------------------------------------------
// Readout (step a6): O[s, i] = sum_k Q[s, k] S_t[i, k]. CTA = 64 tokens x TILE
// output columns of one frame; each thread owns 4 tokens x (TILE/16) columns.
// ----------------------------------------------------------------------------
template <typename T, int TILE>
__global__ void __launch_bounds__(256)
    k_readout_simt(const T* __restrict__ q, const float* __restrict__ Sfr, T* __restrict__ out,
                   int S, int D) {
  constexpr int R = TILE / 16;
  constexpr int TS = 64;
  constexpr int KC = 16;
  __shared__ float Qs[KC][TS + 1];
  __shared__ float Ss[KC][TILE + 1];
  const long long n = blockIdx.x;
  const int s0 = blockIdx.y * TS;
  const int i0 = blockIdx.z * TILE;
  const T* qf = q + (size_t)n * S * D;
  const float* Sn = Sfr + (size_t)n * D * D;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][R];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) acc[a][b] = 0.f;
  for (int k0 = 0; k0 < D; k0 += KC) {
    for (int e = threadIdx.x; e < KC * TS; e += 256) {
      const int tok = e / KC, kk = e % KC, s = s0 + tok;
      Qs[kk][tok] = s < S ? ldf(qf + (size_t)s * D + k0 + kk) : 0.f;
    }
    for (int e = threadIdx.x; e < KC * TILE; e += 256) {
      const int ii = e / KC, kk = e % KC;
      Ss[kk][ii] = Sn[(size_t)(i0 + ii) * D + k0 + kk];
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < KC; ++kk) {
      float qa[4], sb[R];
#pragma unroll
      for (int a = 0; a < 4; ++a) qa[a] = Qs[kk][ty * 4 + a];
#pragma unroll
      for (int b = 0; b < R; ++b) sb[b] = Ss[kk][tx * R + b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < R; ++b) acc[a][b] = fmaf(qa[a], sb[b], acc[a][b]);
    }
    __syncthreads();
  }
  T* of = out + (size_t)n * S * D;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int s = s0 + ty * 4 + a;
    if (s < S)
#pragma unroll
      for (int b = 0; b < R; ++b) stf(of + (size_t)s * D + i0 + tx * R + b, acc[a][b]);
  }
}

template <typename T>
static cudaError_t readout_t(const void* q, const float* Sfr, void* out, long long N, int S,
                             int D, cudaStream_t st) {
  const int tile = D < 64 ? D : 64;
  dim3 grid((unsigned)N, (S + 63) / 64, D / tile);
  switch (tile) {
    case 16:
      k_readout_simt<T, 16><<<grid, 256, 0, st>>>((const T*)q, Sfr, (T*)out, S, D);
      break;
    case 32:
      k_readout_simt<T, 32><<<grid, 256, 0, st>>>((const T*)q, Sfr, (T*)out, S, D);
      break;
    default:
      k_readout_simt<T, 64><<<grid, 256, 0, st>>>((const T*)q, Sfr, (T*)out, S, D);
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t simt_readout(bool bf16, const void* q, const float* Sfr, void* out, long long N,
                         int S, int D, cudaStream_t st) {
  return bf16 ? readout_t<__nv_bfloat16>(q, Sfr, out, N, S, D, st)
              : readout_t<float>(q, Sfr, out, N, S, D, st);
}

}  // namespace gdn
