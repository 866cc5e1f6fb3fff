// Backward pass of the frame-wise GDN scan (CUDA-core kernels).
//
// The pages print no backward; this is the adjoint of the forward recurrence
// (SANA-WM blog, blog.hotdry.top, section 混合线性注意力:
// S_t = gamma_t (S_{t-1} - S_{t-1} A_t) + U_t, O_t = Q_t S_t^T), derived by
// reverse-mode differentiation over the scan order j (frame t_j):
//   G_j  = dO^T Q (frame j) + g_{j+1} (G_{j+1} - G_{j+1} A_{j+1})   (adjoint chain)
//   dQ_t = dO_t S_t,  dM_j = S'_{j}^T G_j  (S'_j: state entering frame j)
//   dA   = -g dM,  dgamma = <dM, I - A>,  dU = G
//   dK^  = diag(beta) (K^ (dA + dA^T) + V G),  dV = diag(beta) K^ G^T
//   dbeta_s = k^_s . (1/2 K^ (dA + dA^T) + V G)_s,  dK = dK^ / sqrt(D S)
// Plan of one call: recompute A_t, U_t and the states S_t (forward kernels),
// W_t = dO_t^T Q_t (the contraction with beta = 1), the adjoint chain for G_t,
// per-frame dM, dA + dA^T and dgamma, then per token the products above.
#include "gdn_internal.cuh"

namespace gdn {

// ----------------------------------------------------------------------------
// dM_j = S'_j^T G_j per frame: S'_j = state_in (j = 0), zeros (reset before
// j), else the stored state after the previous frame in scan order.
// One CTA per (frame, TILE x TILE tile of dM), rows r of S' and G streamed.
// ----------------------------------------------------------------------------
// Element (r, c) of frame f of a matrix array stored as fp32 [F][D][D] or, with
// HILO, as bf16 (hi, lo) pairs [F][2][D][D] (value = hi + lo).
template <bool HILO>
__device__ __forceinline__ float mat_at(const void* base, size_t f, int D, int r, int c) {
  if (HILO) {
    const __nv_bfloat16* b = (const __nv_bfloat16*)base + f * 2 * D * D + (size_t)r * D + c;
    return __bfloat162float(b[0]) + __bfloat162float(b[(size_t)D * D]);
  }
  return ((const float*)base)[f * D * D + (size_t)r * D + c];
}

// Element (k, n) of the D = 128 operand image of A_t (bf16 hi, lo; 128-byte
// swizzled MN-major blocks of 64 columns, hi in bytes [0, 32K), lo after).
__device__ __forceinline__ float img128_at(const uint8_t* img, int k, int n) {
  const int off = (n >> 6) * 16384 + k * 128 + ((((n & 63) >> 3) ^ (k & 7)) << 4) + (n & 7) * 2;
  return __bfloat162float(*(const __nv_bfloat16*)(img + off)) +
         __bfloat162float(*(const __nv_bfloat16*)(img + 32768 + off));
}

template <int TILE, bool HILO>
__global__ void __launch_bounds__(256)
    k_bwd_dm(const void* __restrict__ Sfr, const float* __restrict__ state_in,
             const void* __restrict__ G, float* __restrict__ dM, int T, int D, int reverse,
             int seq_reset, int block) {
  constexpr int R = TILE / 16;
  constexpr int KC = 32;
  __shared__ float Xs[KC][TILE];
  __shared__ float Gs[KC][TILE];
  const long long n = blockIdx.x;
  const int bh = (int)(n / T), t = (int)(n % T);
  const int j = reverse ? T - 1 - t : t;
  // the state entering frame j: state_in (fp32), zeros, or the previous frame's
  const float* X0 = nullptr;
  long long fprev = -1;
  if (j == 0) {
    X0 = state_in ? state_in + (size_t)bh * D * D : nullptr;
  } else {
    const int tp = frame_at(j - 1, T, reverse);
    const bool rst = seq_reset && (t / block) != (tp / block);
    if (!rst) fprev = (long long)bh * T + tp;
  }
  const bool have_x = X0 || fprev >= 0;
  const int nt = D / TILE;
  const int ti = blockIdx.y / nt, tj = blockIdx.y % nt;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[R][R];
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) acc[a][b] = 0.f;
  for (int r0 = 0; have_x && r0 < D; r0 += KC) {
    for (int e = threadIdx.x; e < KC * TILE; e += 256) {
      const int r = e / TILE, c = e % TILE, rr = r0 + r;
      float xv = 0.f, gv = 0.f;
      if (rr < D) {
        xv = X0 ? X0[(size_t)rr * D + ti * TILE + c] : mat_at<HILO>(Sfr, fprev, D, rr, ti * TILE + c);
        gv = mat_at<HILO>(G, n, D, rr, tj * TILE + c);
      }
      Xs[r][c] = xv;
      Gs[r][c] = gv;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < KC; ++r) {
      float xa[R], gb[R];
#pragma unroll
      for (int a = 0; a < R; ++a) {
        xa[a] = Xs[r][ty * R + a];
        gb[a] = Gs[r][tx * R + a];
      }
#pragma unroll
      for (int a = 0; a < R; ++a)
#pragma unroll
        for (int b = 0; b < R; ++b) acc[a][b] = fmaf(xa[a], gb[b], acc[a][b]);
    }
    __syncthreads();
  }
  float* out = dM + (size_t)n * D * D;
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b)
      out[(size_t)(ti * TILE + ty * R + a) * D + tj * TILE + tx * R + b] = acc[a][b];
}

// Per frame, in place: dM -> dA + dA^T = -g (dM + dM^T); dgamma = <dM, I - A>.
// A_t is fp32, or (AIMG, D = 128) its operand image. With `bimg` (D = 128),
// also writes the per-frame B operand of the tensor-core token kernel: bf16
// rows n of [dA + dA^T ; G] (n < 128: dA + dA^T, n >= 128: G row n - 128) by
// 128 columns, K-major, in two 64-column 128-byte-swizzled blocks of 256 rows
// (32 KiB each); G is read from its (hi, lo) pairs and rounded once.
__device__ __forceinline__ int bimg_off(int r, int c) {
  return (c >> 6) * 32768 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + (c & 7) * 2;
}

template <bool AIMG>
__global__ void __launch_bounds__(256)
    k_bwd_dterm(float* __restrict__ dM, const void* __restrict__ A,
                const float* __restrict__ gamma, float* __restrict__ dgamma, int D,
                const __nv_bfloat16* __restrict__ Ghilo, uint8_t* __restrict__ bimg) {
  const long long n = blockIdx.x;
  float* m = dM + (size_t)n * D * D;
  const float* a = AIMG ? nullptr : (const float*)A + (size_t)n * D * D;
  const uint8_t* aimg = AIMG ? (const uint8_t*)A + (size_t)n * D * D * 4 : nullptr;
  uint8_t* bo = bimg ? bimg + (size_t)n * 65536 : nullptr;
  auto a_at = [&](int i, int j) -> float {
    return AIMG ? img128_at(aimg, i, j) : a[(size_t)i * D + j];
  };
  const float g = gamma[n];
  float part = 0.f;
  const int npair = D * (D + 1) / 2;
  for (int e = threadIdx.x; e < npair; e += blockDim.x) {
    // e -> (i, j) with i <= j, row-major over the upper triangle
    int i = 0, rem = e;
    while (rem >= D - i) {
      rem -= D - i;
      ++i;
    }
    const int j = i + rem;
    const float mij = m[(size_t)i * D + j], mji = m[(size_t)j * D + i];
    if (i == j) {
      part += mij * (1.f - a_at(i, i));
      const float s = -2.f * g * mij;
      m[(size_t)i * D + i] = s;
      if (bo) *(__nv_bfloat16*)(bo + bimg_off(i, i)) = __float2bfloat16_rn(s);
    } else {
      part -= (mij + mji) * a_at(i, j);  // A symmetric
      const float s = -g * (mij + mji);
      m[(size_t)i * D + j] = s;
      m[(size_t)j * D + i] = s;
      if (bo) {
        *(__nv_bfloat16*)(bo + bimg_off(i, j)) = __float2bfloat16_rn(s);
        *(__nv_bfloat16*)(bo + bimg_off(j, i)) = __float2bfloat16_rn(s);
      }
    }
  }
  if (bo) {
    const __nv_bfloat16* gh = Ghilo + (size_t)n * 2 * D * D;
    for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
      const int r = e / D, c = e % D;
      const float gv = __bfloat162float(gh[e]) + __bfloat162float(gh[(size_t)D * D + e]);
      *(__nv_bfloat16*)(bo + bimg_off(128 + r, c)) = __float2bfloat16_rn(gv);
    }
  }
  __shared__ float red[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) dgamma[n] = v;
  }
}

// ----------------------------------------------------------------------------
// Token products: out[s, i] = scale sum_k X[s, k] M[i, k]  (M^T; TRANS = 0)
//                                       or X[s, k] M[k, i]  (M;   TRANS = 1)
// per frame n with its own D x D matrix M_n. CTA = 64 tokens x TILE columns.
// ----------------------------------------------------------------------------
template <typename TI, typename TO, int TILE, int TRANS>
__global__ void __launch_bounds__(256)
    k_rowmat_simt(const TI* __restrict__ x, const float* __restrict__ M, TO* __restrict__ out,
                  int S, int D, float scale) {
  constexpr int R = TILE / 16;
  constexpr int TS = 64;
  constexpr int KC = 16;
  __shared__ float Xs[KC][TS + 1];
  __shared__ float Ms[KC][TILE + 1];
  const long long n = blockIdx.x;
  const int s0 = blockIdx.y * TS;
  const int i0 = blockIdx.z * TILE;
  const TI* xf = x + (size_t)n * S * D;
  const float* Mn = M + (size_t)n * D * D;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][R];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) acc[a][b] = 0.f;
  for (int k0 = 0; k0 < D; k0 += KC) {
    for (int e = threadIdx.x; e < KC * TS; e += 256) {
      const int tok = e / KC, kk = e % KC, s = s0 + tok;
      Xs[kk][tok] = s < S ? ldf(xf + (size_t)s * D + k0 + kk) : 0.f;
    }
    for (int e = threadIdx.x; e < KC * TILE; e += 256) {
      const int ii = TRANS ? e % TILE : e / KC, kk = TRANS ? e / TILE : e % KC;
      Ms[kk][ii] = TRANS ? Mn[(size_t)(k0 + kk) * D + i0 + ii] : Mn[(size_t)(i0 + ii) * D + k0 + kk];
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < KC; ++kk) {
      float xa[4], mb[R];
#pragma unroll
      for (int a = 0; a < 4; ++a) xa[a] = Xs[kk][ty * 4 + a];
#pragma unroll
      for (int b = 0; b < R; ++b) mb[b] = Ms[kk][tx * R + b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < R; ++b) acc[a][b] = fmaf(xa[a], mb[b], acc[a][b]);
    }
    __syncthreads();
  }
  TO* of = out + (size_t)n * S * D;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int s = s0 + ty * 4 + a;
    if (s < S)
#pragma unroll
      for (int b = 0; b < R; ++b) stf(of + (size_t)s * D + i0 + tx * R + b, scale * acc[a][b]);
  }
}

template <typename TI, typename TO, int TRANS>
static cudaError_t rowmat(const void* x, const float* M, void* out, long long N, int S, int D,
                          float scale, cudaStream_t st) {
  const int tile = D < 64 ? D : 64;
  dim3 grid((unsigned)N, (S + 63) / 64, D / tile);
  switch (tile) {
    case 16:
      k_rowmat_simt<TI, TO, 16, TRANS><<<grid, 256, 0, st>>>((const TI*)x, M, (TO*)out, S, D, scale);
      break;
    case 32:
      k_rowmat_simt<TI, TO, 32, TRANS><<<grid, 256, 0, st>>>((const TI*)x, M, (TO*)out, S, D, scale);
      break;
    default:
      k_rowmat_simt<TI, TO, 64, TRANS><<<grid, 256, 0, st>>>((const TI*)x, M, (TO*)out, S, D, scale);
  }
  count_launch();
  return cudaGetLastError();
}

// Per token: dk = c beta (P2 + P3), dv = beta P5, dbeta = (c k) . (P2 / 2 + P3),
// with P2 = K^ (dA + dA^T), P3 = V G, P5 = K^ G^T (fp32). One warp per token.
template <typename T>
__global__ void __launch_bounds__(256)
    k_bwd_combine(const T* __restrict__ k, const float* __restrict__ beta,
                  const float* __restrict__ P2, const float* __restrict__ P3,
                  const float* __restrict__ P5, T* __restrict__ dk, T* __restrict__ dv,
                  float* __restrict__ dbeta, long long ntok, int D, float c) {
  const long long tok = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tok >= ntok) return;
  const float b = beta[tok];
  const size_t off = (size_t)tok * D;
  float part = 0.f;
  for (int d = lane; d < D; d += 32) {
    const float p2 = P2[off + d], p3 = P3[off + d], p5 = P5[off + d];
    const float kh = c * ldf(k + off + d);
    stf(dk + off + d, c * b * (p2 + p3));
    stf(dv + off + d, b * p5);
    part = fmaf(kh, 0.5f * p2 + p3, part);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if (lane == 0) dbeta[tok] = part;
}

template <bool HILO>
static cudaError_t bwd_dm_t(const void* Sfr, const float* state_in, const void* G, float* dM,
                            long long N, int T, int D, int reverse, int seq_reset, int block,
                            cudaStream_t st) {
  const int tile = D < 64 ? D : 64;
  dim3 grid((unsigned)N, (D / tile) * (D / tile));
  switch (tile) {
    case 16:
      k_bwd_dm<16, HILO><<<grid, 256, 0, st>>>(Sfr, state_in, G, dM, T, D, reverse, seq_reset, block);
      break;
    case 32:
      k_bwd_dm<32, HILO><<<grid, 256, 0, st>>>(Sfr, state_in, G, dM, T, D, reverse, seq_reset, block);
      break;
    default:
      k_bwd_dm<64, HILO><<<grid, 256, 0, st>>>(Sfr, state_in, G, dM, T, D, reverse, seq_reset, block);
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t simt_bwd_dm(const void* Sfr, const float* state_in, const void* G, float* dM,
                        long long N, int T, int D, int reverse, int seq_reset, int block,
                        bool hilo, cudaStream_t st) {
  return hilo ? bwd_dm_t<true>(Sfr, state_in, G, dM, N, T, D, reverse, seq_reset, block, st)
              : bwd_dm_t<false>(Sfr, state_in, G, dM, N, T, D, reverse, seq_reset, block, st);
}

cudaError_t simt_bwd_dterm(float* dM, const void* A, bool a_image, const float* gamma,
                           float* dgamma, long long N, int D, const void* G_hilo, void* bimg,
                           cudaStream_t st) {
  if (a_image)
    k_bwd_dterm<true><<<(unsigned)N, 256, 0, st>>>(dM, A, gamma, dgamma, D,
                                                   (const __nv_bfloat16*)G_hilo, (uint8_t*)bimg);
  else
    k_bwd_dterm<false><<<(unsigned)N, 256, 0, st>>>(dM, A, gamma, dgamma, D,
                                                    (const __nv_bfloat16*)G_hilo, (uint8_t*)bimg);
  count_launch();
  return cudaGetLastError();
}

// dL/d(state_in) = g_0 (G_0 - G_0 A_0) for the first frame t0 of the scan of
// each head, from G_0 as (hi, lo) pairs and A_0 as its D = 128 operand image.
// CTA = (head, 16 rows); thread (r, l): row r, columns l + 16 m.
__global__ void __launch_bounds__(256)
    k_bwd_ds0(const __nv_bfloat16* __restrict__ Ghilo, const uint8_t* __restrict__ Aimg,
              const float* __restrict__ gamma, float* __restrict__ ds0, int T, int t0) {
  constexpr int D = 128;
  __shared__ float Xs[16][D];
  __shared__ float Ys[16][D];
  const int bh = blockIdx.x, row0 = blockIdx.y * 16;
  const size_t f = (size_t)bh * T + t0;
  const int r = threadIdx.x >> 4, l = threadIdx.x & 15;
  for (int c = l; c < D; c += 16) Xs[r][c] = mat_at<true>(Ghilo, f, D, row0 + r, c);
  float acc[D / 16];
#pragma unroll
  for (int m = 0; m < D / 16; ++m) acc[m] = 0.f;
  const uint8_t* img = Aimg + f * D * D * 4;
  for (int k0 = 0; k0 < D; k0 += 16) {
    __syncthreads();
    for (int e = threadIdx.x; e < 16 * D; e += 256) Ys[e / D][e % D] = img128_at(img, k0 + e / D, e % D);
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < 16; ++kk) {
      const float x = Xs[r][k0 + kk];
#pragma unroll
      for (int m = 0; m < D / 16; ++m) acc[m] = fmaf(x, Ys[kk][l + 16 * m], acc[m]);
    }
  }
  const float g = gamma[f];
#pragma unroll
  for (int m = 0; m < D / 16; ++m) {
    const int c = l + 16 * m;
    ds0[(size_t)bh * D * D + (size_t)(row0 + r) * D + c] = g * (Xs[r][c] - acc[m]);
  }
}

cudaError_t simt_bwd_ds0(const void* G_hilo, const void* A_img, const float* gamma, float* ds0,
                         int heads, int T, int t0, cudaStream_t st) {
  k_bwd_ds0<<<dim3((unsigned)heads, 128 / 16), 256, 0, st>>>((const __nv_bfloat16*)G_hilo,
                                                            (const uint8_t*)A_img, gamma, ds0, T, t0);
  count_launch();
  return cudaGetLastError();
}

cudaError_t simt_rowmat(bool bf16_in, bool f32_out, int trans, const void* x, const float* M,
                        void* out, long long N, int S, int D, float scale, cudaStream_t st) {
  if (bf16_in) {
    if (f32_out)
      return trans ? rowmat<__nv_bfloat16, float, 1>(x, M, out, N, S, D, scale, st)
                   : rowmat<__nv_bfloat16, float, 0>(x, M, out, N, S, D, scale, st);
    return trans ? rowmat<__nv_bfloat16, __nv_bfloat16, 1>(x, M, out, N, S, D, scale, st)
                 : rowmat<__nv_bfloat16, __nv_bfloat16, 0>(x, M, out, N, S, D, scale, st);
  }
  return trans ? rowmat<float, float, 1>(x, M, out, N, S, D, scale, st)
               : rowmat<float, float, 0>(x, M, out, N, S, D, scale, st);
}

cudaError_t simt_bwd_combine(bool bf16, const void* k, const float* beta, const float* P2,
                             const float* P3, const float* P5, void* dk, void* dv, float* dbeta,
                             long long ntok, int D, float c, cudaStream_t st) {
  const unsigned grid = (unsigned)((ntok + 7) / 8);
  if (bf16)
    k_bwd_combine<__nv_bfloat16><<<grid, 256, 0, st>>>(
        (const __nv_bfloat16*)k, beta, P2, P3, P5, (__nv_bfloat16*)dk, (__nv_bfloat16*)dv, dbeta,
        ntok, D, c);
  else
    k_bwd_combine<float><<<grid, 256, 0, st>>>((const float*)k, beta, P2, P3, P5, (float*)dk,
                                               (float*)dv, dbeta, ntok, D, c);
  count_launch();
  return cudaGetLastError();
}

}  // namespace gdn
