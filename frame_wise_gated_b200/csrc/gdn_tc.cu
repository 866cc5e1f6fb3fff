// Tensor-core (tcgen05 / TMEM / TMA) kernels of the frame-wise GDN scan, sm_100a.
//
// Recurrence (SANA-WM blog, blog.hotdry.top, section 混合线性注意力):
//   A_t = K^^T diag(beta_t) K^,  U_t = V_t^T diag(beta_t) K^,  K^ = K / sqrt(D*S)
//   S_t = gamma_t (S_{t-1} - S_{t-1} A_t) + U_t,  O_t = Q_t S_t^T.
//
// k_contract_tc (step a2), D = 128. One CTA per SM, persistent over
// frame-heads. Per 64-token stage, TMA brings K and V tiles ([64 tokens][64 D]
// boxes, 128-byte swizzle) side by side into shared memory; eight scaler warps
// write beta * K in the same layout; one thread issues, per 16 tokens,
//   [A_acc | U_acc^T] += (beta K)^T [K | V]
// as one 128x256x16 bf16 MMA (A_t is symmetric, so (beta K)^T K = A_t).
// (beta K)^T and [K | V] are read as MN-major operands straight from the
// token-major tiles: no transposes. The fp32 accumulators live in TMEM
// (2 x 256 columns, double-buffered so the epilogue of one frame-head overlaps
// the MMAs of the next); four epilogue warps scale them (1/(D S) and
// 1/sqrt(D S)) and store A_t (row by row) and U_t (column by column).
//
// k_readout_tc (step a6), D = 128. Per 128-token tile of a frame-head,
//   O_tile = Q_tile S_t^T = Q_tile S_hi^T + Q_tile S_lo^T
// with S_t held as a bf16 (hi, lo) pair (the pair carries ~16 bits of the
// fp32 state). Q tiles stream through a 3-stage TMA ring, the accumulator is
// double-buffered in TMEM, and the epilogue converts to bf16 into a swizzled
// staging tile that one thread writes back with a TMA store.
//
// Every wait is bounded (see sm100::mbar_wait); a wait that runs out records
// a status the host reads with gdn_check_device_status.
#include <cuda.h>

#include <mutex>

#include "gdn_internal.cuh"
#include "gdn_sm100.cuh"

namespace gdn {

static __device__ int g_tc_status = 0;

using namespace sm100;

// ----------------------------------------------------------------------------
// host: tensor maps through the driver entry point (no link-time libcuda)
// ----------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  });
  return fn;
}

// 3-D bf16 tensor [d2][d1][d0] (d0 innermost), box {b0, b1, 1}, 128-byte swizzle.
static cudaError_t make_map_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1,
                                    uint64_t d2, uint32_t b0, uint32_t b1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

static int num_sms() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// Kernel attributes such as the dynamic shared-memory limit belong to the
// kernel as loaded on one device, so each launch site sets them once per
// device: one bit per device, a mutex for concurrent host threads.
struct DeviceOnce {
  std::mutex mu;
  unsigned long long done = 0;
};

template <class F>
static cudaError_t once_per_device(DeviceOnce& o, F&& set) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(o.mu);
  if ((o.done >> dev) & 1ull) return cudaSuccess;
  e = set();
  if (e == cudaSuccess) o.done |= 1ull << dev;
  return e;
}

// Rounds the dynamic shared-memory base up to 1024 bytes (the 128-byte
// swizzle atom repeats every 1024). The offset is added to the pointer itself,
// so the compiler still knows the result addresses shared memory and emits
// shared-memory loads and stores for it rather than generic ones.
__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// One arrival per warp on `bar` (initialised with a count of warps), after
// every lane's own fences: 32 lanes arriving one by one serialise on the
// barrier word.
__device__ __forceinline__ void warp_arrive(uint32_t bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// ----------------------------------------------------------------------------
// Prologue inside the loaders (SANA-WM blog, Context-Parallel section: the
// fused op runs RMSNorm -> ReLU -> key scale -> RoPE ahead of the scan), D = 128.
// Each thread takes NR token rows rr[] of a tile made of two [rows][64] bf16
// boxes with the 128-byte swizzle, and in each row the 32 channels of its
// quarter q (channels 32q .. 32q + 31: four 16-byte chunks); the four threads
// that share a row combine their sums of squares. Lane layout (pro_lane): a
// warp holds 8 rows; lane 8q + j takes quarter q of row j. Each 8-lane phase
// of a 16-byte access then covers 8 rows of one quarter, whose swizzled
// chunks fall in 8 distinct bank groups: no bank conflicts. With
// NR = 2 the rows run side by side so that the latency of one (shared-memory
// loads, shuffles, rsqrt) overlaps the arithmetic of the other. Since the RMSNorm
// factor inv = 1/sqrt(mean(x^2) + eps) is positive and RoPE is linear,
//     RoPE(max(x * inv * w, 0)) = inv * RoPE(max(x * w, 0)),
// so inv scales the rotated pair. The rows are written back in place; with
// `btile`, bv[k] * row k also goes to `btile` (same layout).
//
// Weights come from shared memory laid out by pro_w_copy: w4[p * 4 + q] =
// (w[32q + 2p], w[32q + 2p + 1]), so the four quarters' threads of a warp read
// 32 adjacent bytes. RoPE: pair i of a half (i < 32) turns by pos * theta_i,
// pos the token's row (channels below 64) or column (above). With `theta`
// (shared memory, the 32 frequencies) the (cos, sin) is computed by
// rope_cs_reduced. Otherwise it is read from `tab`, a shared copy of the
// table laid out by pro_table_index. THETA and BTILE are template flags so
// that the unrolled pair loop holds no branches.
// ----------------------------------------------------------------------------
// Frequency of pair i of an axis half of D/2 channels: base^(-2i/(D/2)).
__device__ __forceinline__ float rope_theta(float base, int i, int D) {
  return powf(base, -2.0f * (float)i / (float)(D / 2));
}

// (cos, sin) of ang = pos * theta for the hardware sine/cosine, which is
// accurate only near zero. The angle is first brought to [-pi, pi] by
// Cody-Waite reduction (W. J. Cody and W. Waite, "Software Manual for the
// Elementary Functions", 1980): k = rint(ang / 2pi), then ang - k * C1 - k * C2
// with 2pi = C1 + C2, C1 the fp32 nearest 2pi and C2 the remainder. Each step
// is a fused multiply-add, rounded once on a result already near zero, so C1
// needs no shortened mantissa. The error is then about 1e-6 plus the fp32
// rounding of pos * theta (2^-24 of the angle), below the bf16 rounding the
// prologue's result gets.
__device__ __forceinline__ float2 rope_cs_reduced(int pos, float theta) {
  float ang = (float)pos * theta;
  const float k = rintf(ang * 0.159154943091895f);  // 1 / (2 pi)
  ang = fmaf(-k, 6.28318548202514648f, ang);         // C1 = 2 pi rounded to fp32
  ang = fmaf(-k, -1.7484555314695172e-7f, ang);      // C2 = 2 pi - C1
  float2 cs;
  __sincosf(ang, &cs.y, &cs.x);
  return cs;
}

constexpr int PRO_POS_PITCH = 80;  // positions per pair in the shared table (the most supported)
__device__ __forceinline__ int pro_table_index(int i, int pos) {
  // pairs i and i + 16 of one position are neighbours, positions of one pair
  // are consecutive: the threads of a warp (8 tokens x 4 quarters) read
  // 16 consecutive entries in the column half and 2 in the row half. The
  // fixed pitch makes the pair offsets compile-time constants.
  return (((i & 15) * PRO_POS_PITCH + pos) << 1) + (i >> 4);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Row (of the warp's 8, plus 8 per warp before it) and quarter of thread t.
__device__ __forceinline__ int pro_lane_row(int t) { return ((t >> 5) << 3) + (t & 7); }
__device__ __forceinline__ int pro_lane_quarter(int t) { return (t >> 3) & 3; }

// The prologue with the camera encoding (SANA-WM blog, section 双分支相机控制:
// each token's transform into its ray-local frame, combined with the RoPE on
// separate channels): channels 0-63 (box 0) form 16 blocks of 4, each
// multiplied by the token's 4 x 4 matrix (pro.ucpe at frame-head n); channels
// 64-127 (box 1) carry the 2-D RoPE of a 64-channel vector, y on channels
// 64-95 and x on 96-127, 16 pairs each (table / theta entries 0-15). RMSNorm,
// ReLU and the beta * K^ copy as in pro_rows.
// Threads keep pro_rows' layout for the sum of squares (lane 8 q + j: quarter
// q of row j). For the transform every lane takes the same work, so a warp
// never splits between the two kinds: 16-byte chunks 2q and 2q + 1 of box 0
// (two camera blocks each) and of box 1 (eight RoPE pairs). The lanes of a row
// read its raw chunks before __syncwarp, then write. The matrices come from
// global memory (L2: the heads of a frame share them); rows past S clamp to
// token S - 1 (their data are zeros).
template <int NR, bool THETA, bool BTILE>
__device__ __forceinline__ void pro_rows_ucpe(uint8_t* tile, int box_bytes, const int (&rr)[NR],
                                              int q, const int (&tk)[NR], int S,
                                              const ProArgs& pro, const float2* w4,
                                              const float2* tab, const float* theta,
                                              uint8_t* btile, const float (&bv)[NR], int n) {
  constexpr int D = 128;
  auto chunk_off = [&](int box, int row, int ch) {
    return box * box_bytes + row * 128 + ((ch ^ (row & 7)) << 4);
  };
  float inv[NR], scb[NR];
  {
    float ss[NR];
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 v = *(const uint4*)(tile + chunk_off(q >> 1, rr[k], (q & 1) * 4 + c));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = unpack_bf16x2(w[e]);
          acc = __ffma2_rn(x, x, acc);
        }
      }
      ss[k] = acc.x + acc.y;
    }
#pragma unroll
    for (int o = 8; o < 32; o <<= 1) {  // the row's four quarters: lanes j, j + 8, j + 16, j + 24
#pragma unroll
      for (int k = 0; k < NR; ++k) ss[k] += __shfl_xor_sync(0xffffffffu, ss[k], o);
    }
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      inv[k] = rsqrtf(fmaf(ss[k], 1.0f / (float)D, pro.eps));
      scb[k] = inv[k] * bv[k];
    }
  }
  // this lane's raw chunks: camera chunks 2q, 2q + 1 of box 0, RoPE chunks of box 1
  uint32_t cw[NR][8], rw[NR][8];
#pragma unroll
  for (int k = 0; k < NR; ++k)
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 a = *(const uint4*)(tile + chunk_off(0, rr[k], 2 * q + i));
      const uint4 b = *(const uint4*)(tile + chunk_off(1, rr[k], 2 * q + i));
      cw[k][4 * i] = a.x; cw[k][4 * i + 1] = a.y; cw[k][4 * i + 2] = a.z; cw[k][4 * i + 3] = a.w;
      rw[k][4 * i] = b.x; rw[k][4 * i + 1] = b.y; rw[k][4 * i + 2] = b.z; rw[k][4 * i + 3] = b.w;
    }
  __syncwarp();  // the lanes of each row have read their raw chunks
  // camera: chunk ch = 2q + i of box 0 holds channels 8 ch .. 8 ch + 7 (quarter
  // ch / 4, words 4 (ch % 4) .. + 3 of it): blocks 2 ch and 2 ch + 1
  const long long bt = (long long)(n / (pro.H * pro.T)) * pro.T + n % pro.T;
#pragma unroll
  for (int k = 0; k < NR; ++k) {
    const int s = tk[k] < S ? tk[k] : S - 1;
    const float4* mp = (const float4*)(pro.ucpe + ((size_t)bt * S + s) * 16);
    const float4 m0 = __ldg(mp), m1 = __ldg(mp + 1), m2 = __ldg(mp + 2), m3 = __ldg(mp + 3);
    // the matrix by column pairs, the RMSNorm factor folded in: output rows
    // (0, 1) are sum_j c01[j] v_j and rows (2, 3) sum_j c23[j] v_j (packed fp32x2)
    const float f = inv[k];
    const float2 c01[4] = {make_float2(m0.x * f, m1.x * f), make_float2(m0.y * f, m1.y * f),
                           make_float2(m0.z * f, m1.z * f), make_float2(m0.w * f, m1.w * f)};
    const float2 c23[4] = {make_float2(m2.x * f, m3.x * f), make_float2(m2.y * f, m3.y * f),
                           make_float2(m2.z * f, m3.z * f), make_float2(m2.w * f, m3.w * f)};
    const float bq = BTILE ? bv[k] : 1.f;  // beta: scb / inv
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int ch = 2 * q + i, qc = ch >> 2, pw = 4 * (ch & 3);
      uint32_t ow[4], obw[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 x0 = __fmul2_rn(unpack_bf16x2(cw[k][4 * i + 2 * h]), w4[(pw + 2 * h) * 4 + qc]);
        const float2 x1 =
            __fmul2_rn(unpack_bf16x2(cw[k][4 * i + 2 * h + 1]), w4[(pw + 2 * h + 1) * 4 + qc]);
        const float v0 = fmaxf(x0.x, 0.f), v1 = fmaxf(x0.y, 0.f), v2 = fmaxf(x1.x, 0.f),
                    v3 = fmaxf(x1.y, 0.f);
        float2 o01 = __fmul2_rn(c01[0], make_float2(v0, v0));
        float2 o23 = __fmul2_rn(c23[0], make_float2(v0, v0));
        o01 = __ffma2_rn(c01[1], make_float2(v1, v1), o01);
        o23 = __ffma2_rn(c23[1], make_float2(v1, v1), o23);
        o01 = __ffma2_rn(c01[2], make_float2(v2, v2), o01);
        o23 = __ffma2_rn(c23[2], make_float2(v2, v2), o23);
        o01 = __ffma2_rn(c01[3], make_float2(v3, v3), o01);
        o23 = __ffma2_rn(c23[3], make_float2(v3, v3), o23);
        ow[2 * h] = pack_bf16x2(o01.x, o01.y);
        ow[2 * h + 1] = pack_bf16x2(o23.x, o23.y);
        if (BTILE) {
          const float2 b01 = __fmul2_rn(o01, make_float2(bq, bq));
          const float2 b23 = __fmul2_rn(o23, make_float2(bq, bq));
          obw[2 * h] = pack_bf16x2(b01.x, b01.y);
          obw[2 * h + 1] = pack_bf16x2(b23.x, b23.y);
        }
      }
      const int off = chunk_off(0, rr[k], ch);
      *(uint4*)(tile + off) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      if (BTILE) *(uint4*)(btile + off) = make_uint4(obw[0], obw[1], obw[2], obw[3]);
    }
  }
  // RoPE: chunk ch = 2q + i of box 1 is quarter 2 + ch / 4 (y for ch < 4, x
  // after), words 4 (ch % 4) .. + 3 = pairs of the same index
#pragma unroll
  for (int k = 0; k < NR; ++k) {
    const int pos = tk[k] < S ? ((q >> 1) ? tk[k] % pro.grid_w : tk[k] / pro.grid_w) : 0;
    const float2* trow = tab + pro_table_index(0, pos);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int ch = 2 * q + i, qr = 2 + (ch >> 2), pw = 4 * (ch & 3);
      uint32_t ow[4], obw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int p = pw + e;
        const float2 m = __fmul2_rn(unpack_bf16x2(rw[k][4 * i + e]), w4[p * 4 + qr]);
        const float a = fmaxf(m.x, 0.f), b = fmaxf(m.y, 0.f);
        const float2 t = THETA ? rope_cs_reduced(pos, theta[p]) : trow[p * 2 * PRO_POS_PITCH];
        const float2 o = make_float2(a * t.x - b * t.y, a * t.y + b * t.x);
        ow[e] = pack_bf16x2(o.x * inv[k], o.y * inv[k]);
        if (BTILE) obw[e] = pack_bf16x2(o.x * scb[k], o.y * scb[k]);
      }
      const int off = chunk_off(1, rr[k], ch);
      *(uint4*)(tile + off) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      if (BTILE) *(uint4*)(btile + off) = make_uint4(obw[0], obw[1], obw[2], obw[3]);
    }
  }
}

template <int NR, bool THETA, bool BTILE>
__device__ __forceinline__ void pro_rows_rope(uint8_t* tile, int box_bytes, const int (&rr)[NR],
                                              int q, const int (&tk)[NR], int S,
                                              const ProArgs& pro, const float2* w4,
                                              const float2* tab, const float* theta,
                                              uint8_t* btile, const float (&bv)[NR]) {
  constexpr int D = 128, NW = 16;  // channel pairs (packed words) per thread row
  const int box = q >> 1, ch0 = (q & 1) * 4, pb = (q & 1) * 16;
  uint32_t u[NR][NW];
#pragma unroll
  for (int k = 0; k < NR; ++k)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = *(const uint4*)(tile + box * box_bytes + rr[k] * 128 +
                                      (((ch0 + c) ^ (rr[k] & 7)) << 4));
      u[k][4 * c] = v.x;
      u[k][4 * c + 1] = v.y;
      u[k][4 * c + 2] = v.z;
      u[k][4 * c + 3] = v.w;
    }
  float inv[NR], scb[NR];
  int pos[NR];
  const float2* trow[NR];  // table entries of the rows' positions (pair pb + p at p * 2 * pitch)
  {
    float2 acc[NR][2];
#pragma unroll
    for (int k = 0; k < NR; ++k) acc[k][0] = acc[k][1] = make_float2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < NW; ++e)
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        const float2 x = unpack_bf16x2(u[k][e]);
        acc[k][e & 1] = __ffma2_rn(x, x, acc[k][e & 1]);
      }
    float ss[NR];
#pragma unroll
    for (int k = 0; k < NR; ++k) ss[k] = (acc[k][0].x + acc[k][0].y) + (acc[k][1].x + acc[k][1].y);
#pragma unroll
    for (int o = 8; o < 32; o <<= 1) {  // the row's four quarters: lanes j, j + 8, j + 16, j + 24
      float sh[NR];
#pragma unroll
      for (int k = 0; k < NR; ++k) sh[k] = __shfl_xor_sync(0xffffffffu, ss[k], o);
#pragma unroll
      for (int k = 0; k < NR; ++k) ss[k] += sh[k];
    }
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      inv[k] = rsqrtf(fmaf(ss[k], 1.0f / (float)D, pro.eps));
      scb[k] = inv[k] * bv[k];
      pos[k] = tk[k] < S ? (box ? tk[k] % pro.grid_w : tk[k] / pro.grid_w) : 0;
      trow[k] = tab + pro_table_index(pb, pos[k]);
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t ob[NR][4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int p = 4 * c + e;  // pair p of the thread: pair pb + p of its half
      const float2 w2 = w4[p * 4 + q];
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        const float2 m = __fmul2_rn(unpack_bf16x2(u[k][p]), w2);
        const float a = fmaxf(m.x, 0.f), b = fmaxf(m.y, 0.f);
        float2 t;
        if (THETA) {
          t = rope_cs_reduced(pos[k], theta[pb + p]);
        } else {
          t = trow[k][p * 2 * PRO_POS_PITCH];
        }
        const float2 o = make_float2(a * t.x - b * t.y, a * t.y + b * t.x);
        const float2 kh = __fmul2_rn(o, make_float2(inv[k], inv[k]));
        u[k][p] = pack_bf16x2(kh.x, kh.y);
        if (BTILE) {
          const float2 bk = __fmul2_rn(o, make_float2(scb[k], scb[k]));
          ob[k][e] = pack_bf16x2(bk.x, bk.y);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      const int off = box * box_bytes + rr[k] * 128 + (((ch0 + c) ^ (rr[k] & 7)) << 4);
      *(uint4*)(tile + off) = make_uint4(u[k][4 * c], u[k][4 * c + 1], u[k][4 * c + 2], u[k][4 * c + 3]);
      if (BTILE) *(uint4*)(btile + off) = make_uint4(ob[k][0], ob[k][1], ob[k][2], ob[k][3]);
    }
  }
}

// The prologue of NR rows; UC (the camera encoding) is a compile-time choice so
// that the kernels without it keep their register allocation.
template <int NR, bool THETA, bool BTILE, bool UC>
__device__ __forceinline__ void pro_rows(uint8_t* tile, int box_bytes, const int (&rr)[NR], int q,
                                         const int (&tk)[NR], int S, const ProArgs& pro,
                                         const float2* w4, const float2* tab, const float* theta,
                                         uint8_t* btile, const float (&bv)[NR], int n) {
  if constexpr (UC)
    pro_rows_ucpe<NR, THETA, BTILE>(tile, box_bytes, rr, q, tk, S, pro, w4, tab, theta, btile, bv,
                                    n);
  else
    pro_rows_rope<NR, THETA, BTILE>(tile, box_bytes, rr, q, tk, S, pro, w4, tab, theta, btile, bv);
}

// Fills the shared (cos, sin) table in pro_table_index order: entry (i, pos)
// holds the turn of pair i at position pos, pos * base^(-2i/(Dr/2)) for the
// RoPE's Dr channels (128, or 64 with the camera encoding), by
// rope_cs_reduced (the bidirectional readout's function). Each CTA computes
// its own copy at start-up (a few thousand entries over all its threads), so
// no separate table launch precedes the kernel.
__device__ __forceinline__ void pro_table_fill(float2* tab, const ProArgs& pro) {
  const int dr = pro.ucpe ? 64 : 128;
  const int npairs = dr / 4;
  for (int e = threadIdx.x; e < pro.npos * npairs; e += (int)blockDim.x) {
    const int i = e / pro.npos, pos = e - i * pro.npos;
    tab[pro_table_index(i, pos)] = rope_cs_reduced(pos, rope_theta(pro.base, i, dr));
  }
}

// Copies the RMSNorm weights w[128] into shared memory in pro_rows' order.
__device__ __forceinline__ void pro_w_copy(float2* w4, const float* w) {
  for (int e = threadIdx.x; e < 64; e += (int)blockDim.x) {
    const int p = e & 15, q = e >> 4;
    w4[p * 4 + q] = make_float2(w[32 * q + 2 * p], w[32 * q + 2 * p + 1]);
  }
}

// (cos, sin) of pos * base^(-2i/(D/2)) for pos < npos, i < D/4, at cs[i * npos + pos].
__global__ void k_rope_table(float2* cs, int npos, int D, float base) {
  const int n = npos * (D / 4);
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
    const int i = e / npos, pos = e % npos;
    const float theta = rope_theta(base, i, D);
    float sn, c;
    sincosf((float)pos * theta, &sn, &c);
    cs[e] = make_float2(c, sn);
  }
}

// The same layout as k_rope_table, through rope_cs_reduced (the path the
// bidirectional readout's prologue takes); for tests of its accuracy.
__global__ void k_rope_reduced(float2* cs, int npos, int D, float base) {
  const int n = npos * (D / 4);
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
    const int i = e / npos, pos = e % npos;
    cs[e] = rope_cs_reduced(pos, rope_theta(base, i, D));
  }
}

cudaError_t rope_table(float2* cs, int npos, int D, float base, cudaStream_t st) {
  const int n = npos * (D / 4);
  k_rope_table<<<(n + 255) / 256, 256, 0, st>>>(cs, npos, D, base);
  count_launch();
  return cudaGetLastError();
}

cudaError_t rope_reduced(float2* cs, int npos, int D, float base, cudaStream_t st) {
  const int n = npos * (D / 4);
  k_rope_reduced<<<(n + 255) / 256, 256, 0, st>>>(cs, npos, D, base);
  count_launch();
  return cudaGetLastError();
}

// ============================================================================
// Contraction (a2)
// ============================================================================
namespace ctr {
constexpr int D = 128;
constexpr int TOK = 64;                 // tokens per stage
constexpr int BOX = TOK * 128;          // one [64 tokens][64 channels] bf16 box: 8 KiB
constexpr int TILE = 2 * BOX;           // one tensor's stage tile: 16 KiB
constexpr int TAB_MAX = PRO_POS_PITCH * 32;  // prologue table entries: positions x pairs (D/4 = 32)
constexpr int NSC = 256;                // scaler threads (8 warps)
constexpr int THREADS = 64 + NSC + 128;  // producer, MMA, 8 scaler warps, 4 epilogue warps
constexpr uint32_t TMEM_COLS = 512;
constexpr int NST_PLAIN = 6;
constexpr int NST_PRO = 4;
// Shared-memory layout for an NST-stage K/V ring: 6 stages and 2 beta * K
// slots without the prologue; with it, 4 stages, 4 slots and the (cos, sin)
// table. The two scaler groups take alternate stages, so with 4 slots a group
// starts its next stage while the MMAs of its last one still read their slot.
template <int NST>
struct Lay {
  static constexpr int NBK = NST == NST_PRO ? 4 : 2;  // beta * K slots (the MMA's B operand)
  static constexpr int OFF_K = 0;                     // stage s: K at s * 2 TILE, V after it
  static constexpr int OFF_BK = OFF_K + NST * 2 * TILE;
  static constexpr int OFF_BETA = OFF_BK + NBK * TILE;
  static constexpr int OFF_BAR = OFF_BETA + NST * TOK * 4;
  // full, empty per stage; bk_full, bk_empty per slot; acc_full[2], acc_empty[2], fin
  static constexpr int NBAR = 2 * NST + 2 * NBK + 5;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_TAB = OFF_MISC + 16;
  static constexpr int SMEM_PLAIN = OFF_TAB + 1024;
  static constexpr int OFF_W4 = OFF_TAB + TAB_MAX * 8;  // prologue weights (pro_w_copy order)
  static constexpr int SMEM_PRO = OFF_W4 + 512 + 1024;
};
constexpr int SMEM_PLAIN = Lay<NST_PLAIN>::SMEM_PLAIN;
constexpr int SMEM_PRO = Lay<NST_PRO>::SMEM_PRO;
static_assert(SMEM_PLAIN <= 232448 && SMEM_PRO <= 232448, "contraction shared memory");
}  // namespace ctr

// Bounded wait until the shared counter *c reaches `target`; false on abort or
// when 2 s run out (the timeout is recorded with `code`).
__device__ __forceinline__ bool wait_count_ge(volatile int* c, int target, volatile int* abort_flag,
                                              int code) {
  if (*c >= target) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (*c >= target) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > kWaitNs) {
        atomicCAS(&g_tc_status, 0, code);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Frame-head n's A_t image (discard & 2) and U_t (discard & 1) are read once, by
// its chain, which then adds a fifth count to flags[n]. Once that count is
// there, epilogue warp q drops its quarter of their L2 lines without a write
// back. With `wait` the warp polls for the count for at most 100 us; otherwise
// it looks once. A line that is not dropped is simply written back later.
__device__ __forceinline__ void drop_consumed(float* A, float* U, const int* flags, int n, int q,
                                             int lane, int discard, int wait) {
  int ok = 0;
  if (lane == 0) {
    const unsigned long long t0 = wait ? globaltimer() : 0ull;
    for (;;) {
      int v;
      asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(flags + n) : "memory");
      if (v >= 5) {
        ok = 1;
        break;
      }
      if (!wait || globaltimer() - t0 > 100000ull) break;
      __nanosleep(256);
    }
  }
  if (!__shfl_sync(0xffffffffu, ok, 0)) return;
  const size_t base = (size_t)n * kImageBytes + (size_t)q * (kImageBytes / 4);
#pragma unroll
  for (int j = 0; j < 4; ++j) {  // 4 lines of 128 bytes per lane: the warp's 16 KiB quarter
    const size_t off = base + (size_t)(j * 32 + lane) * 128;
    if (discard & 2) discard_l2_line((const uint8_t*)A + off);
    if (discard & 1) discard_l2_line((const uint8_t*)U + off);
  }
}

// Body of the contraction for CTA `cta` of `ncta` contraction CTAs. Units are
// frame-heads in order n, or, when `heads` > 0, in scan order across heads
// (unit u -> head u % heads, scan position u / heads of T: frame u / heads, or
// T - 1 - u / heads when `rev`). With `flags`, each of the 4 epilogue warps
// publishes its rows of A_t, U_t by a release increment of flags[n], so a
// concurrent scan may read frame-head n once flags[n] reaches 4. Warps beyond
// the contraction's 14 (when the block is larger) only join the barriers.
//
// Rings: K and V tiles in NST stages (freed by the MMA commit of the stage),
// beta * K in NBK slots of its own (written by the scalers once the MMAs of
// the stage NBK earlier are done), so the ring that waits on HBM is deep.
template <int NST, bool UC = false>
__device__ __forceinline__ void contract_body(const CUtensorMap& tmK, const CUtensorMap& tmV,
                                              const float* __restrict__ beta, float* __restrict__ A,
                                              float* __restrict__ U, int N, int S, float cA,
                                              float cU, int a_image, const ProArgs& pro, int cta,
                                              int ncta, int heads, int T, int rev, int* flags,
                                              int parts = 1, int discard = 0) {
  using namespace ctr;
  using Ly = Lay<NST>;
  constexpr int NBK = Ly::NBK;
  constexpr int OFF_K = Ly::OFF_K, OFF_BK = Ly::OFF_BK, OFF_BETA = Ly::OFF_BETA;
  constexpr int OFF_MISC = Ly::OFF_MISC, OFF_TAB = Ly::OFF_TAB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_full = sb + Ly::OFF_BAR;
  const uint32_t bar_empty = bar_full + 8 * NST;
  const uint32_t bar_bkf = bar_empty + 8 * NST;
  const uint32_t bar_bke = bar_bkf + 8 * NBK;
  const uint32_t bar_accf = bar_bke + 8 * NBK;
  const uint32_t bar_acce = bar_accf + 16;
  const uint32_t bar_fin = bar_acce + 16;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  volatile int* mma_issued = (volatile int*)(smem + OFF_MISC + 8);  // stages the MMA has issued

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full + 8 * s, 33);     // expect_tx arrival + 32 lanes' beta copies
      mbar_init(bar_empty + 8 * s, 1);     // MMA commit
    }
    for (int s = 0; s < NBK; ++s) {
      mbar_init(bar_bkf + 8 * s, NSC / 64);  // every warp of the slot's scaler group
      mbar_init(bar_bke + 8 * s, 1);        // MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf + 8 * b, 1);
      mbar_init(bar_acce + 8 * b, 4);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    *mma_issued = 0;
    fence_mbar_init();
  }
  float2* tab = (float2*)(smem + OFF_TAB);
  float2* w4 = (float2*)(smem + Ly::OFF_W4);
  if (pro.w) {
    pro_table_fill(tab, pro);
    pro_w_copy(w4, pro.w);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int nst_frame = (S + TOK - 1) / TOK;
  // parts > 1: each frame-head's tokens are cut into `parts` stage ranges, one
  // unit each, whose partial A_t, U_t are added (fp32 atomics) into A, U. The
  // ranges are balanced, part * nst / parts .. (part + 1) * nst / parts, so
  // none is empty while parts <= nst (the host keeps parts <= nst / 2): an
  // empty unit would add a stale TMEM accumulator into A_t, U_t.
  const int NU = N * parts;
  const int my_count = cta < NU ? (NU - 1 - cta) / ncta + 1 : 0;
  auto unit_n = [&](int i) -> int {
    const int u = (cta + i * ncta) / parts;
    if (heads <= 0) return u;
    const int j = u / heads;
    return (u % heads) * T + (rev ? T - 1 - j : j);
  };
  auto st_begin = [&](int i) -> int { return ((cta + i * ncta) % parts) * nst_frame / parts; };
  auto st_end = [&](int i) -> int { return ((cta + i * ncta) % parts + 1) * nst_frame / parts; };

  // Stages of beta * K are taken by groups of 4 warps (128 threads each,
  // four threads per token with the prologue: tokens pr and pr + 32 of the
  // stage). Two scaler groups alternate stages. With the prologue, whose
  // arithmetic sets the pace, the 4 epilogue warps (busy only once per unit)
  // form a third group: a unit's first 8 stages alternate between groups 0
  // and 1, later stages rotate over all three, so the epilogue's drain of
  // the previous unit at the start of a unit holds up no early stage.
  constexpr bool EPI3 = NST == NST_PRO;
  auto stage_owner = [&](int i, int st, int g) -> int {
    if (!EPI3) return g & 1;
    const int r = st - st_begin(i);
    return r < 8 ? (r & 1) : (r - 8) % 3;
  };
  // One stage by one group (tt = 0..127); false if a wait ran out.
  auto scale_stage = [&](int i, int st, int g, int tt) -> bool {
    const int pr = pro_lane_row(tt), pq = pro_lane_quarter(tt);
    const int s = g % NST, kb = g % NBK;
    const uint32_t u = (uint32_t)(g / NST);
    // Stage s and slot kb pass between groups, and their barriers are waited
    // on by parity, which tells only the last two phases apart: with three
    // groups, first let the MMA issue the previous uses of both (stages
    // g - NST and g - NBK). Then the wanted phase is the next one on each.
    constexpr int PREV = NST < NBK ? NST : NBK;
    if (EPI3 && !wait_count_ge(mma_issued, g - PREV + 1, abort_flag, 9)) return false;
    bool ok = mbar_wait(bar_full + 8 * s, u & 1, abort_flag, &g_tc_status, 6);
    // the slot's previous beta * K has been consumed by its MMAs
    if (ok) ok = mbar_wait(bar_bke + 8 * kb, ((uint32_t)(g / NBK) & 1) ^ 1, abort_flag, &g_tc_status, 8);
    if (!ok) return false;
    uint8_t* kt = smem + OFF_K + s * 2 * TILE;
    uint8_t* bt = smem + OFF_BK + kb * TILE;
    const float* bs = (const float*)(smem + OFF_BETA) + s * TOK;
    if (pro.w) {
      // raw k -> K^ in place (RMSNorm, ReLU, RoPE) and beta * K^ into the slot
      const int rr[2] = {pr, pr + 32}, tk[2] = {st * TOK + pr, st * TOK + pr + 32};
      const float bv[2] = {beta ? bs[pr] : 1.f, beta ? bs[pr + 32] : 1.f};
      pro_rows<2, false, true, UC>(kt, BOX, rr, pq, tk, S, pro, w4, tab, nullptr, bt, bv,
                                   unit_n(i));
      fence_proxy_async();
      warp_arrive(bar_bkf + 8 * kb);
      return true;
    }
#pragma unroll
    for (int m = 0; m < 1024 / (NSC / 2); ++m) {
      const int c = tt + (NSC / 2) * m;   // 16-byte chunk of the 16 KiB tile
      const float bv = beta ? bs[(c >> 3) & (TOK - 1)] : 1.f;  // 8 chunks per 128-byte token row
      uint4 x = *(const uint4*)(kt + c * 16);
      uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&w[e]);
        float2 f = __bfloat1622float2(h);
        w[e] = pack_bf16x2(f.x * bv, f.y * bv);
      }
      *(uint4*)(bt + c * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    fence_proxy_async();
    warp_arrive(bar_bkf + 8 * kb);
    return true;
  };

  if (warp == 0) {
    // ---- TMA producer (lane 0 issues; the warp loads beta) ----
    int g = 0;
    bool ok = true;
    for (int i = 0; i < my_count && ok; ++i) {
      const int n = unit_n(i);
      for (int st = st_begin(i); st < st_end(i); ++st, ++g) {
        const int s = g % NST;
        const uint32_t u = (uint32_t)(g / NST);
        if (lane == 0) ok = mbar_wait(bar_empty + 8 * s, (u & 1) ^ 1, abort_flag, &g_tc_status, 1);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          // K and V are read once: evict-first keeps L2 for the A_t, U_t and
          // state lines that the chains read back
          const uint64_t pol = l2_policy_evict_first();
          const uint32_t kd = sb + OFF_K + s * 2 * TILE, vd = kd + TILE;
          mbar_arrive_expect_tx(bar_full + 8 * s, 2 * TILE);
          tma_load_3d_hint(kd, &tmK, bar_full + 8 * s, 0, st * TOK, n, pol);
          tma_load_3d_hint(kd + BOX, &tmK, bar_full + 8 * s, 64, st * TOK, n, pol);
          tma_load_3d_hint(vd, &tmV, bar_full + 8 * s, 0, st * TOK, n, pol);
          tma_load_3d_hint(vd + BOX, &tmV, bar_full + 8 * s, 64, st * TOK, n, pol);
        }
        // beta of the stage's tokens: asynchronous 4-byte copies (zeros past S)
        // that arrive on the same barrier, so the loop never waits on them.
        const uint32_t bsa = sb + OFF_BETA + s * TOK * 4;
        if (beta) {
#pragma unroll
          for (int r = lane; r < TOK; r += 32) {
            const int tok = st * TOK + r;
            const bool in = tok < S;
            cp_async_4(bsa + r * 4, beta + (size_t)n * S + (in ? tok : 0), in ? 4u : 0u);
          }
          cp_async_arrive_noinc(bar_full + 8 * s);
        } else {
          mbar_arrive(bar_full + 8 * s);  // beta = 1: nothing to copy
        }
      }
    }
    // Drain: every TMA this CTA issued has landed before teardown.
    if (lane == 0) {
      for (int gg = (g > NST ? g - NST : 0); gg < g; ++gg)
        mbar_wait(bar_full + 8 * (gg % NST), (uint32_t)(gg / NST) & 1, abort_flag, &g_tc_status, 2);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256, true, true);
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_count && ok; ++i) {
        const int b = i & 1;
        const uint32_t ub = (uint32_t)(i >> 1);
        ok = mbar_wait(bar_acce + 8 * b, (ub & 1) ^ 1, abort_flag, &g_tc_status, 3);
        if (!ok) break;
        tc_fence_after();
        const uint32_t dAU = tmem + b * 256;
        const int st0 = st_begin(i);
        for (int st = st0; st < st_end(i); ++st, ++g) {
          const int s = g % NST, kb = g % NBK;
          ok = mbar_wait(bar_bkf + 8 * kb, (uint32_t)(g / NBK) & 1, abort_flag, &g_tc_status, 4);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kva = sb + OFF_K + s * 2 * TILE, ba = sb + OFF_BK + kb * TILE;
#pragma unroll
          for (int kk = 0; kk < TOK / 16; ++kk) {
            // 16 tokens = two 8-row groups of 1024 B; [K | V] is one N = 256
            // operand of four 64-channel blocks
            const uint64_t dkv = smem_desc_sw128(kva + kk * 2048, BOX, 1024);
            const uint64_t db = smem_desc_sw128(ba + kk * 2048, BOX, 1024);
            const uint32_t acc = (st > st0 || kk > 0) ? 1u : 0u;
            mma_bf16(dAU, db, dkv, idesc, acc);
          }
          mma_commit(bar_empty + 8 * s);
          mma_commit(bar_bke + 8 * kb);
          if (EPI3) *mma_issued = g + 1;
        }
        if (!ok) break;
        mma_commit(bar_accf + 8 * b);
      }
      mma_commit(bar_fin);
      mbar_wait(bar_fin, 0, abort_flag, &g_tc_status, 5);
    }
    __syncwarp();
  } else if (warp < 2 + NSC / 32) {
    // ---- beta * K into the B operand tile (same swizzled layout as K) ----
    const int t = threadIdx.x - 64;
    const int grp = t >> 7, tt = t & 127;
    int g = 0;
    bool ok = true;
    for (int i = 0; i < my_count && ok; ++i) {
      for (int st = st_begin(i); st < st_end(i); ++st, ++g) {
        if (stage_owner(i, st, g) != grp) continue;
        if (!scale_stage(i, st, g, tt)) {
          ok = false;
          break;
        }
      }
    }
  } else if (warp < 2 + NSC / 32 + 4) {
    // ---- epilogue: TMEM -> scale -> fp32 A_t, U_t rows ----
    const int q = warp & 3;
    const int row = q * 32 + lane;
    // unit i's accumulator out of TMEM; false if a wait ran out
    auto epi = [&](int i) -> bool {
      const int b = i & 1;
      const uint32_t ub = (uint32_t)(i >> 1);
      // lane 0 waits and the warp follows its decision (warp-uniform control flow)
      int ok = 1;
      if (lane == 0) ok = mbar_wait(bar_accf + 8 * b, ub & 1, abort_flag, &g_tc_status, 7);
      if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
      __syncwarp();
      tc_fence_after();
      const int n = unit_n(i);
#pragma unroll
      for (int half = a_image == 2 ? 1 : 0; half < 2; ++half) {  // 2: only U is wanted
        float* dst = (half ? U : A) + ((size_t)n * D + row) * D;
        uint8_t* img = (uint8_t*)A + (size_t)n * kImageBytes;
        const float sc = half ? cU : cA;
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + b * 256 + half * 128 + c0, r);
          tmem_wait_ld();
          if (parts > 1) {
            // partial sums: row `row` of A_t (fp32, 16-byte atomics); column
            // `row` of U_t (each warp adds 32 consecutive floats per row)
            if (half == 0) {
#pragma unroll
              for (int j = 0; j < 8; ++j)
                atomicAdd((float4*)(dst + c0 + 4 * j),
                          make_float4(__uint_as_float(r[4 * j]) * sc, __uint_as_float(r[4 * j + 1]) * sc,
                                      __uint_as_float(r[4 * j + 2]) * sc, __uint_as_float(r[4 * j + 3]) * sc));
            } else {
              float* ucol = U + (size_t)n * D * D + row;
#pragma unroll
              for (int j = 0; j < 32; ++j) atomicAdd(ucol + (size_t)(c0 + j) * D, __uint_as_float(r[j]) * sc);
            }
          } else if (half == 0 && a_image) {
            // A_t row `row` as the B-operand image (row k = row, columns c0..c0+31)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int col = c0 + 8 * j;
              uint32_t hw[4], lw[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float a0 = __uint_as_float(r[8 * j + 2 * e]) * sc;
                const float a1 = __uint_as_float(r[8 * j + 2 * e + 1]) * sc;
                const __nv_bfloat16 h0 = __float2bfloat16_rn(a0), h1 = __float2bfloat16_rn(a1);
                hw[e] = pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
                lw[e] = pack_bf16x2(a0 - __bfloat162float(h0), a1 - __bfloat162float(h1));
              }
              const int off = (col >> 6) * (128 * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4);
              *(uint4*)(img + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              *(uint4*)(img + 32768 + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
          } else if (half == 0) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              float4 v = make_float4(__uint_as_float(r[4 * j]) * sc, __uint_as_float(r[4 * j + 1]) * sc,
                                     __uint_as_float(r[4 * j + 2]) * sc,
                                     __uint_as_float(r[4 * j + 3]) * sc);
              *(float4*)(dst + c0 + 4 * j) = v;
            }
          } else {
            // TMEM holds U_t^T (lane = key channel `row`, column = value
            // channel): column `row` of U_t, rows c0..c0+31; the warp's 32
            // lanes store 32 consecutive floats of each row
            float* ucol = U + (size_t)n * D * D + row;
#pragma unroll
            for (int j = 0; j < 32; ++j) ucol[(size_t)(c0 + j) * D] = __uint_as_float(r[j]) * sc;
          }
        }
      }
      tc_fence_before();
      warp_arrive(bar_acce + 8 * b);
      if (flags) {
        // publish this warp's rows of A_t, U_t: its stores, made visible to
        // other CTAs' bulk/TMA loads (async proxy), then a release increment
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
        __syncwarp();
        if (lane == 0)
          asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(flags + n), "r"(1) : "memory");
        // the previous unit's A_t image and U_t, once its chain has copied them
        // (count 5: 4 publications + 1 consumption), are never read again
        if (discard && i > 0) drop_consumed(A, U, flags, unit_n(i - 1), q, lane, discard, 0);
      }
      return true;
    };
    if (EPI3) {
      // third scaler group: drain the previous unit, then take this unit's stages
      const int tt = threadIdx.x - (64 + NSC);
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_count && ok; ++i) {
        if (i > 0 && !epi(i - 1)) {
          ok = false;
          break;
        }
        for (int st = st_begin(i); st < st_end(i); ++st, ++g) {
          if (stage_owner(i, st, g) != 2) continue;
          if (!scale_stage(i, st, g, tt)) {
            ok = false;
            break;
          }
        }
      }
      if (ok && my_count > 0) epi(my_count - 1);
    } else {
      for (int i = 0; i < my_count; ++i)
        if (!epi(i)) break;
    }
    // this CTA's last unit: its chain reads it shortly; wait for that a while
    if (discard && my_count > 0) drop_consumed(A, U, flags, unit_n(my_count - 1), q, lane, discard, 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int NST, bool UC = false>
__global__ void __launch_bounds__(ctr::THREADS, 1)
    k_contract_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const float* __restrict__ beta, float* __restrict__ A, float* __restrict__ U,
                  int N, int S, float cA, float cU, int a_image, ProArgs pro, int parts) {
  contract_body<NST, UC>(tmK, tmV, beta, A, U, N, S, cA, cU, a_image, pro, blockIdx.x, gridDim.x, 0, 0,
                     0, nullptr, parts);
}

bool tc_contract_supported(int D) { return D == 128 || D == 64 || D == 256; }

// Token-split contraction (D = 128) for problems with few frame-heads: each
// frame-head's tokens are cut into `parts` ranges on separate CTAs whose
// partial A_t, U_t are added into the zeroed fp32 Aacc, U (the caller turns
// Aacc into operand images afterwards).
static cudaError_t tc_contract128(const void* k, const void* v, const float* beta, float* A,
                                  float* U, long long N, int S, int D, float cA, float cU,
                                  int a_image, const ProArgs* pro, cudaStream_t st, int parts);
cudaError_t tc_contract_split(const void* k, const void* v, const float* beta, float* Aacc,
                              float* U, long long N, int S, float cA, float cU, int parts,
                              const ProArgs* pro, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(Aacc, 0, (size_t)N * 128 * 128 * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(U, 0, (size_t)N * 128 * 128 * 4, st);
  if (e != cudaSuccess) return e;
  return tc_contract128(k, v, beta, Aacc, U, N, S, 128, cA, cU, 0, pro, st, parts);
}
int tc_prologue_max_positions() { return ctr::TAB_MAX / 32; }

static cudaError_t tc_contract128(const void* k, const void* v, const float* beta, float* A,
                                  float* U, long long N, int S, int D, float cA, float cU,
                                  int a_image, const ProArgs* pro, cudaStream_t st, int parts = 1) {
  if (D != 128) return cudaErrorNotSupported;
  if (pro && pro->npos * (D / 4) > ctr::TAB_MAX) return cudaErrorNotSupported;
  ProArgs pa = {};
  if (pro) pa = *pro;
  CUtensorMap mk, mv;
  cudaError_t e = make_map_bf16_3d(&mk, k, D, S, N, 64, ctr::TOK);
  if (e != cudaSuccess) return e;
  e = make_map_bf16_3d(&mv, v, D, S, N, 64, ctr::TOK);
  if (e != cudaSuccess) return e;
  static DeviceOnce attr_once;
  const cudaError_t attr_status = once_per_device(attr_once, [&]() -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(k_contract_tc<ctr::NST_PLAIN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ctr::SMEM_PLAIN);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_contract_tc<ctr::NST_PRO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               ctr::SMEM_PRO);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_contract_tc<ctr::NST_PRO, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, ctr::SMEM_PRO);
    return e;
  });
  if (attr_status != cudaSuccess) return attr_status;
  const long long units = N * parts;
  const int grid = (int)(units < num_sms() ? units : num_sms());
  if (pro && pro->ucpe)
    k_contract_tc<ctr::NST_PRO, true><<<grid, ctr::THREADS, ctr::SMEM_PRO, st>>>(
        mk, mv, beta, A, U, (int)N, S, cA, cU, a_image, pa, parts);
  else if (pro)
    k_contract_tc<ctr::NST_PRO><<<grid, ctr::THREADS, ctr::SMEM_PRO, st>>>(
        mk, mv, beta, A, U, (int)N, S, cA, cU, a_image, pa, parts);
  else
    k_contract_tc<ctr::NST_PLAIN><<<grid, ctr::THREADS, ctr::SMEM_PLAIN, st>>>(
        mk, mv, beta, A, U, (int)N, S, cA, cU, a_image, pa, parts);
  count_launch();
  return cudaGetLastError();
}

// ============================================================================
// Readout (a6)
// ============================================================================
namespace rdo {
constexpr int D = 128;
constexpr int TOK = 128;                // tokens per tile (MMA M)
constexpr int NQ = 3;                   // Q ring stages
constexpr int BOX = TOK * 128;          // [128 rows][64 channels] bf16: 16 KiB
constexpr int QT = 2 * BOX;             // one Q tile: 32 KiB
constexpr int OFF_Q = 0;
constexpr int OFF_S = OFF_Q + NQ * QT;  // S hi (2 boxes) then S lo (2 boxes): 64 KiB
constexpr int OFF_O = OFF_S + 4 * BOX;  // output staging, 2 boxes: 32 KiB
constexpr int OFF_BAR = OFF_O + 2 * BOX;
constexpr int NBAR = 3 * NQ + 2 + 4 + 1;  // q_full, q_ready, q_empty, s_full, s_empty, acc f/e x2, fin
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int OFF_TAB = OFF_MISC + 16;  // prologue (cos, sin) table copy
constexpr int TAB_MAX = PRO_POS_PITCH * 32;
constexpr int OFF_W4 = OFF_TAB + TAB_MAX * 8;  // prologue weights (pro_w_copy order)
constexpr int SMEM = OFF_W4 + 512 + 1024;
// producer, MMA, 4 epilogue warps (+ 8 warps applying the prologue to Q tiles)
constexpr int threads(bool pro) { return pro ? 448 : 192; }
constexpr uint32_t TMEM_COLS = 256;
}  // namespace rdo

// TRANS: O = Q S_t (S_t as an MN-major operand) instead of Q S_t^T; the
// backward's dQ = dO S_t.
template <bool PRO, bool TRANS = false, bool UC = false>
__global__ void __launch_bounds__(rdo::threads(PRO), 1)
    k_readout_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmS,
                 const __grid_constant__ CUtensorMap tmO, int N, int S, ProArgs pro, int parts) {
  using namespace rdo;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_qf = sb + OFF_BAR;
  const uint32_t bar_qr = bar_qf + 8 * NQ;  // Q tile transformed by the prologue warps
  const uint32_t bar_qe = bar_qr + 8 * NQ;
  const uint32_t bar_sf = bar_qe + 8 * NQ;
  const uint32_t bar_se = bar_sf + 8;
  const uint32_t bar_accf = bar_se + 8;
  const uint32_t bar_acce = bar_accf + 16;
  const uint32_t bar_fin = bar_acce + 16;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NQ; ++s) {
      mbar_init(bar_qf + 8 * s, 1);
      mbar_init(bar_qr + 8 * s, 8);  // every prologue warp
      mbar_init(bar_qe + 8 * s, 1);
    }
    mbar_init(bar_sf, 1);
    mbar_init(bar_se, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf + 8 * b, 1);
      mbar_init(bar_acce + 8 * b, 4);  // every epilogue warp
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (PRO) {
    pro_table_fill((float2*)(smem + OFF_TAB), pro);
    pro_w_copy((float2*)(smem + OFF_W4), pro.w);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int ntile = (S + TOK - 1) / TOK;
  // Work units: each frame-head's tiles in kParts contiguous parts (outputs are
  // per token, so parts need no reduction); finer units even out the rounds.
  const int kParts = parts;
  const int NU = N * kParts;
  const int my_count = (int)blockIdx.x < NU ? (NU - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp == 0) {
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_count && ok; ++i) {
        const int unit = blockIdx.x + i * gridDim.x;
        const int n = unit / kParts, part = unit % kParts;
        const int tl0 = part * ntile / kParts, tl1 = (part + 1) * ntile / kParts;
        (void)n;
                ok = mbar_wait(bar_se, ((uint32_t)i & 1) ^ 1, abort_flag, &g_tc_status, 11);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_sf, 4 * BOX);
        const uint32_t sd = sb + OFF_S;
        tma_load_3d(sd, &tmS, bar_sf, 0, 0, 2 * n);
        tma_load_3d(sd + BOX, &tmS, bar_sf, 64, 0, 2 * n);
        tma_load_3d(sd + 2 * BOX, &tmS, bar_sf, 0, 0, 2 * n + 1);
        tma_load_3d(sd + 3 * BOX, &tmS, bar_sf, 64, 0, 2 * n + 1);
        for (int tl = tl0; tl < tl1; ++tl, ++g) {
          const int s = g % NQ;
          const uint32_t u = (uint32_t)(g / NQ);
          ok = mbar_wait(bar_qe + 8 * s, (u & 1) ^ 1, abort_flag, &g_tc_status, 12);
          if (!ok) break;
          const uint32_t qd = sb + OFF_Q + s * QT;
          mbar_arrive_expect_tx(bar_qf + 8 * s, QT);
          tma_load_3d(qd, &tmQ, bar_qf + 8 * s, 0, tl * TOK, n);
          tma_load_3d(qd + BOX, &tmQ, bar_qf + 8 * s, 64, tl * TOK, n);
        }
      }
      for (int gg = (g > NQ ? g - NQ : 0); gg < g; ++gg)
        mbar_wait(bar_qf + 8 * (gg % NQ), (uint32_t)(gg / NQ) & 1, abort_flag, &g_tc_status, 13);
      if (my_count > 0) mbar_wait(bar_sf, (uint32_t)(my_count - 1) & 1, abort_flag, &g_tc_status, 14);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, TRANS);
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_count && ok; ++i) {
        const int unit = blockIdx.x + i * gridDim.x;
        const int n = unit / kParts, part = unit % kParts;
        const int tl0 = part * ntile / kParts, tl1 = (part + 1) * ntile / kParts;
        (void)n;
        ok = mbar_wait(bar_sf, (uint32_t)i & 1, abort_flag, &g_tc_status, 15);
        if (!ok) break;
        tc_fence_after();
        for (int tl = tl0; tl < tl1; ++tl, ++g) {
          const int s = g % NQ;
          const uint32_t u = (uint32_t)(g / NQ);
          const int b = g & 1;
          const uint32_t ub = (uint32_t)(g >> 1);
          ok = mbar_wait(bar_acce + 8 * b, (ub & 1) ^ 1, abort_flag, &g_tc_status, 16);
          if (!ok) break;
          ok = mbar_wait((PRO ? bar_qr : bar_qf) + 8 * s, u & 1, abort_flag, &g_tc_status, 17);
          if (!ok) break;
          tc_fence_after();
          const uint32_t qa = sb + OFF_Q + s * QT, sh = sb + OFF_S, sl = sb + OFF_S + 2 * BOX;
          const uint32_t d = tmem + b * 128;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            // K-major: 16 channels = 32 bytes inside a 128-byte swizzled row
            const uint32_t off = (kk >> 2) * BOX + (kk & 3) * 32;
            const uint64_t dq = smem_desc_sw128(qa + off, 16, 1024);
            // S_t^T: K-major rows of S_t; S_t: 16 rows of k, two 64-column blocks
            const uint64_t dh = TRANS ? smem_desc_sw128(sh + kk * 2048, BOX, 1024)
                                      : smem_desc_sw128(sh + off, 16, 1024);
            const uint64_t dl = TRANS ? smem_desc_sw128(sl + kk * 2048, BOX, 1024)
                                      : smem_desc_sw128(sl + off, 16, 1024);
            mma_bf16(d, dq, dh, idesc, kk > 0 ? 1u : 0u);
            mma_bf16(d, dq, dl, idesc, 1u);
          }
          mma_commit(bar_qe + 8 * s);
          mma_commit(bar_accf + 8 * b);
        }
        if (!ok) break;
        mma_commit(bar_se);
      }
      mma_commit(bar_fin);
      mbar_wait(bar_fin, 0, abort_flag, &g_tc_status, 18);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ---- epilogue: TMEM -> bf16 -> swizzled staging -> TMA store ----
    const int q = warp & 3;
    const int row = q * 32 + lane;  // token within the tile
    const int et = threadIdx.x - 64;
    uint8_t* ost = smem + OFF_O;
    const uint32_t ost_a = sb + OFF_O;
    int g = 0;
    bool ok = true;
    for (int i = 0; i < my_count && ok; ++i) {
      const int unit = blockIdx.x + i * gridDim.x;
      const int n = unit / kParts, part = unit % kParts;
      const int tl0 = part * ntile / kParts, tl1 = (part + 1) * ntile / kParts;
      (void)n;
            for (int tl = tl0; tl < tl1; ++tl, ++g) {
        const int b = g & 1;
        const uint32_t ub = (uint32_t)(g >> 1);
        mbar_wait(bar_accf + 8 * b, ub & 1, abort_flag, &g_tc_status, 19);
        tc_fence_after();
        // the previous tile's TMA store has finished reading the staging tile
        if (et == 0) bulk_wait_read0();
        // one decision for all four epilogue warps: the flag may be set while they read it
        if (named_bar_or(1, 128, *abort_flag != 0)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t packed[32];
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + b * 128 + half * 64 + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j)
              packed[c0 / 2 + j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
          }
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint8_t* dst = ost + half * BOX + row * 128 + ((c ^ (row & 7)) << 4);
            *(uint4*)dst = make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2],
                                      packed[4 * c + 3]);
          }
        }
        tc_fence_before();
        warp_arrive(bar_acce + 8 * b);
        fence_proxy_async();
        named_bar_sync(1, 128);
        if (et == 0) {
          tma_store_3d(&tmO, ost_a, 0, tl * TOK, n);
          tma_store_3d(&tmO, ost_a + BOX, 64, tl * TOK, n);
          bulk_commit();
        }
      }
    }
    if (et == 0) bulk_wait0();
  } else if (PRO) {
    // ---- prologue on each raw Q tile, in place: four threads per token
    // (32 channels each), tokens pr and pr + 64 ----
    const int t = threadIdx.x - 192;
    const int pr = pro_lane_row(t), pq = pro_lane_quarter(t);
    int g = 0;
    bool ok = true;
    for (int i = 0; i < my_count && ok; ++i) {
      const int unit = blockIdx.x + i * gridDim.x;
      const int n = unit / kParts, part = unit % kParts;
      const int tl0 = part * ntile / kParts, tl1 = (part + 1) * ntile / kParts;
      (void)n;
      for (int tl = tl0; tl < tl1; ++tl, ++g) {
        const int s = g % NQ;
        const uint32_t u = (uint32_t)(g / NQ);
        ok = mbar_wait(bar_qf + 8 * s, u & 1, abort_flag, &g_tc_status, 20);
        if (!ok) break;
        const int rr[2] = {pr, pr + 64}, tk[2] = {tl * TOK + pr, tl * TOK + pr + 64};
        const float bv[2] = {1.f, 1.f};
        pro_rows<2, false, false, UC>(smem + OFF_Q + s * QT, BOX, rr, pq, tk, S, pro,
                                  (const float2*)(smem + OFF_W4), (const float2*)(smem + OFF_TAB),
                                  nullptr, nullptr, bv, n);
        fence_proxy_async();
        warp_arrive(bar_qr + 8 * s);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

bool tc_readout_supported(int D) { return D == 128 || D == 64 || D == 256; }

// Readout work units: each frame-head's tiles in three contiguous parts when
// a part still holds four tiles or more and there are fewer than 32 rounds
// of frame-heads (finer units even out the last round of the persistent grid;
// measured on 720p frames, 29 tiles: 3 parts beat 1, 2 and 4 for 48, 336 and
// 1936 frame-heads; with 7808 the extra state loads cost more than they
// save), else two when there are fewer than four rounds.
static int readout_parts(long long N, int ntile) {
  if (ntile >= 12 && N < 32LL * num_sms()) return 3;
  return (ntile >= 8 && N < 4LL * num_sms()) ? 2 : 1;
}

template <bool PRO, bool TRANS = false, bool UC = false>
static cudaError_t launch_readout(const CUtensorMap& mq, const CUtensorMap& ms, const CUtensorMap& mo,
                                  long long N, int S, const ProArgs& pa, cudaStream_t st) {
  static DeviceOnce attr_once;
  const cudaError_t attr_status = once_per_device(attr_once, [&]() -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(k_readout_tc<PRO, TRANS, UC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         rdo::SMEM);
    return e;
  });
  if (attr_status != cudaSuccess) return attr_status;
  const int parts = readout_parts(N, (S + rdo::TOK - 1) / rdo::TOK);
  const long long units = N * parts;
  const int grid = (int)(units < num_sms() ? units : num_sms());
  k_readout_tc<PRO, TRANS, UC><<<grid, rdo::threads(PRO), rdo::SMEM, st>>>(mq, ms, mo, (int)N, S,
                                                                          pa, parts);
  count_launch();
  return cudaGetLastError();
}

static cudaError_t tc_readout128(const void* q, const void* Sfr_hilo, void* out, long long N,
                                 int S, int D, const ProArgs* pro, cudaStream_t st) {
  if (D != 128) return cudaErrorNotSupported;
  if (pro && pro->npos * (D / 4) > rdo::TAB_MAX) return cudaErrorNotSupported;
  CUtensorMap mq, ms, mo;
  cudaError_t e = make_map_bf16_3d(&mq, q, D, S, N, 64, rdo::TOK);
  if (e != cudaSuccess) return e;
  e = make_map_bf16_3d(&ms, Sfr_hilo, D, D, 2 * N, 64, 128);
  if (e != cudaSuccess) return e;
  e = make_map_bf16_3d(&mo, out, D, S, N, 64, rdo::TOK);
  if (e != cudaSuccess) return e;
  ProArgs pa = {};
  if (pro) {
    pa = *pro;
    if (pa.ucpe) return launch_readout<true, false, true>(mq, ms, mo, N, S, pa, st);
    return launch_readout<true>(mq, ms, mo, N, S, pa, st);
  }
  return launch_readout<false>(mq, ms, mo, N, S, pa, st);
}

// dQ_t = dO_t S_t for every frame-head (D = 128, bf16; S_t as bf16 hi/lo pairs).
cudaError_t tc_readout_trans(const void* x, const void* Sfr_hilo, void* out, long long N, int S,
                             cudaStream_t st) {
  CUtensorMap mq, ms, mo;
  cudaError_t e = make_map_bf16_3d(&mq, x, 128, S, N, 64, rdo::TOK);
  if (e == cudaSuccess) e = make_map_bf16_3d(&ms, Sfr_hilo, 128, 128, 2 * N, 64, 128);
  if (e == cudaSuccess) e = make_map_bf16_3d(&mo, out, 128, S, N, 64, rdo::TOK);
  if (e != cudaSuccess) return e;
  ProArgs pa = {};
  return launch_readout<false, true>(mq, ms, mo, N, S, pa, st);
}

// ============================================================================
// Chains of the recurrence on tensor cores (steps a3, a4, a5), D = 128.
//
// One CTA runs one chain X <- alpha (X - X Y) + Z (the state update; the span
// composites E <- E + A - E A and H <- gamma (H - H A) + U; the prefix over
// spans S <- g (S - S E) + H). The 128 x 128 fp32 X lives in registers: warp
// w holds rows 32 (w % 4) .. +31 (its TMEM lane quadrant), columns
// 64 (w / 4) .. +63. Each step writes X as a bf16 (hi, lo) pair into a K-major
// operand tile and one thread issues
//     P = X_hi Y_hi + X_lo Y_hi + X_hi Y_lo      (fp32 in TMEM)
// which carries ~16 mantissa bits of both factors. Y (fp32 in global memory)
// is split into bf16 (hi, lo) MN-major tiles for the next step while the
// current step's MMAs run (two Y buffers).
// ============================================================================
namespace chn {
constexpr int D = 128;
constexpr int HALF = 64 * 128 * 2 * 2;  // one bf16 128x128 operand tile: 32 KiB
constexpr int ATOM = 128 * 128;         // 16 KiB: 128 rows x 128 bytes
constexpr int OFF_XH = 0;
constexpr int OFF_XL = OFF_XH + HALF;
constexpr int OFF_Y = OFF_XL + HALF;     // Y operand image (hi, then lo)
constexpr int OFF_Z = OFF_Y + kImageBytes;  // Z fp32: 4 boxes of [128 rows][32 fp32], swizzled
constexpr int OFF_BAR = OFF_Z + kImageBytes;  // bar_mma, bar_y, bar_z
constexpr int OFF_MISC = OFF_BAR + 32;
constexpr int SMEM = OFF_MISC + 16 + 1024;
constexpr int THREADS = 256;
constexpr uint32_t TMEM_COLS = 128;
}  // namespace chn

struct ChainStep {
  const void* Y;    // operand image of Y
  const float* Z;   // fp32 Z, or null: Z = Y (span composite E)
  float alpha;
  int reset;        // zero X before this step
  int t;            // frame (scan/compose) or span (prefix)
};

// Program of chain c: number of steps and, for step s, its operands.
struct ChainProg {
  int mode, which, bh, p, j0, n;
  const float* init;
  int init_hilo;  // init points at a bf16 (hi, lo) pair
};

__device__ __forceinline__ ChainProg chain_prog(const ChainArgs& a, int c) {
  ChainProg g;
  g.mode = a.mode;
  g.which = 0;
  g.init = nullptr;
  g.init_hilo = 0;
  if (a.mode == CHAIN_SCAN) {
    g.bh = c / a.nseg;
    g.p = c % a.nseg;
    int j0, j1;
    seg_range(a, g.p, &j0, &j1);
    g.j0 = j0;
    g.n = j1 - j0;
    if (g.p == 0)
      g.init = a.state_in ? a.state_in + (size_t)g.bh * a.D * a.D : nullptr;
    else if (a.seg == SEG_CHUNKS) {
      g.init = a.Sst + ((size_t)g.bh * a.nseg + g.p) * a.D * a.D;
      g.init_hilo = a.sst_hilo;
    }
  } else if (a.mode == CHAIN_COMPOSE) {
    const int half = a.heads * a.nseg;
    g.which = c >= half;
    const int cc = g.which ? c - half : c;
    g.bh = cc / a.nseg;
    g.p = cc % a.nseg;
    int j0, j1;
    seg_range(a, g.p, &j0, &j1);
    g.j0 = j0;
    g.n = j1 - j0;
  } else if (a.mode == CHAIN_ADJOINT) {
    // backward: one chain per head over the scan positions T-1 .. 0, starting
    // from the gradient of state_out
    g.bh = c;
    g.p = 0;
    g.j0 = 0;
    g.n = a.T;
    g.init = a.dS_out ? a.dS_out + (size_t)g.bh * a.D * a.D : nullptr;
  } else {
    g.bh = c;
    g.p = 0;
    g.j0 = 0;
    g.n = a.nseg - 1;
    g.init = a.state_in ? a.state_in + (size_t)g.bh * a.D * a.D : nullptr;
  }
  return g;
}

__device__ __forceinline__ ChainStep chain_step_at(const ChainArgs& a, const ChainProg& g, int s) {
  ChainStep st;
  const size_t DD = (size_t)a.D * a.D;
  if (g.mode == CHAIN_PREFIX) {
    const size_t si = (size_t)g.bh * a.nseg + s;
    st.Y = a.E + si * DD;
    st.Z = a.Hc + si * DD;
    st.alpha = a.g[si];
    st.reset = 0;
    st.t = s;
    return st;
  }
  if (g.mode == CHAIN_ADJOINT) {
    // G_j = W_j + g_{j+1} (G_{j+1} - G_{j+1} A_{j+1}), cut where the forward
    // scan reset before j+1; the first step (j = T-1) only adds W.
    const int j = a.T - 1 - s;
    const int t = frame_at(j, a.T, a.reverse);
    st.t = t;
    st.Z = a.Zw + ((size_t)g.bh * a.T + t) * DD;
    st.reset = 0;
    if (s == 0) {
      st.Y = a.zero_img;
      st.alpha = 1.0f;
    } else {
      const int tn = frame_at(j + 1, a.T, a.reverse);
      const size_t fn = (size_t)g.bh * a.T + tn;
      st.Y = a.A + fn * DD;
      st.alpha = a.gamma[fn];
      st.reset = a.seq_reset && (t / a.block) != (tn / a.block);
    }
    return st;
  }
  const int j = g.j0 + s;
  const int t = frame_at(j, a.T, a.reverse);
  const size_t fi = (size_t)g.bh * a.T + t;
  st.t = t;
  st.Y = a.A + fi * DD;
  st.reset = 0;
  if (g.mode == CHAIN_SCAN) {
    st.Z = a.U + fi * DD;
    st.alpha = a.gamma[fi];
    if (a.seg == SEG_SEQUENTIAL && a.seq_reset && j > 0) {
      const int tp = frame_at(j - 1, a.T, a.reverse);
      st.reset = (t / a.block) != (tp / a.block);
    }
  } else {
    st.Z = g.which ? a.U + fi * DD : nullptr;
    st.alpha = g.which ? a.gamma[fi] : 1.0f;
  }
  return st;
}

// Bulk copy of one operand image (64 KiB) into shared memory; one thread.
__device__ __forceinline__ void chain_fetch_y(uint32_t dst, const void* src, uint32_t bar) {
  mbar_arrive_expect_tx(bar, kImageBytes);
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"((uint32_t)kImageBytes), "r"(bar)
      : "memory");
}

// X row slice (64 values of row `row`, columns 64h..) -> hi/lo 16-byte chunks
// at `off(c)` of tiles xh / xl (c = chunk 0..7 of the slice).
__device__ __forceinline__ void split_chunk(const float* v, uint4* hi, uint4* lo) {
  uint32_t hw[4], lw[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float a0 = v[2 * e], a1 = v[2 * e + 1];
    const __nv_bfloat16 h0 = __float2bfloat16_rn(a0), h1 = __float2bfloat16_rn(a1);
    hw[e] = pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
    lw[e] = pack_bf16x2(a0 - __bfloat162float(h0), a1 - __bfloat162float(h1));
  }
  *hi = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  *lo = make_uint4(lw[0], lw[1], lw[2], lw[3]);
}

// Same swizzled position for K-major X tiles (rows = state rows, 64 columns per
// 128-byte row of atom h) and for MN-major operand images (rows = k, 64
// columns n per 128-byte row of block h).
__device__ __forceinline__ int tile_off(int row, int h, int c) {
  return h * chn::ATOM + row * 128 + ((c ^ (row & 7)) << 4);
}

__device__ __forceinline__ void chain_store_x(const float* x, uint8_t* xh, uint8_t* xl, int row,
                                              int h) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 hi, lo;
    split_chunk(x + 8 * c, &hi, &lo);
    *(uint4*)(xh + tile_off(row, h, c)) = hi;
    *(uint4*)(xl + tile_off(row, h, c)) = lo;
  }
}

// 64 values of row `row`, columns 64h.., of an initial state: fp32, or a bf16
// (hi, lo) pair whose hi matrix starts at `init` (lo follows D*D values later).
__device__ __forceinline__ void load_init_slice(const float* init, int hilo, int row, int h,
                                                float* x) {
  constexpr int D = chn::D;
  if (!init) {
#pragma unroll
    for (int c = 0; c < 64; ++c) x[c] = 0.f;
  } else if (hilo) {
    const __nv_bfloat16* hi = (const __nv_bfloat16*)init + (size_t)row * D + h * 64;
    const __nv_bfloat16* lo = hi + (size_t)D * D;
#pragma unroll
    for (int c = 0; c < 64; c += 8) {
      const uint4 a4 = __ldg((const uint4*)(hi + c)), b4 = __ldg((const uint4*)(lo + c));
      const uint32_t aw[4] = {a4.x, a4.y, a4.z, a4.w}, bw[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[e]));
        const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bw[e]));
        x[c + 2 * e] = fa.x + fb.x;
        x[c + 2 * e + 1] = fa.y + fb.y;
      }
    }
  } else {
    const float* src = init + (size_t)row * D + h * 64;
#pragma unroll
    for (int c = 0; c < 64; c += 4) {
      const float4 f = __ldg((const float4*)(src + c));
      x[c] = f.x; x[c + 1] = f.y; x[c + 2] = f.z; x[c + 3] = f.w;
    }
  }
}

__device__ __forceinline__ void store_row_f32(float* dst, const float* x) {
#pragma unroll
  for (int c = 0; c < 64; c += 4) *(float4*)(dst + c) = make_float4(x[c], x[c + 1], x[c + 2], x[c + 3]);
}

__device__ __forceinline__ void store_row_hilo(__nv_bfloat16* hi, __nv_bfloat16* lo, const float* x) {
#pragma unroll
  for (int c = 0; c < 64; c += 8) split_chunk(x + c, (uint4*)(hi + c), (uint4*)(lo + c));
}

__device__ __forceinline__ void store_row_image(uint8_t* img, const float* x, int row, int h) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    split_chunk(x + 8 * c, (uint4*)(img + tile_off(row, h, c)),
                (uint4*)(img + 2 * chn::ATOM + tile_off(row, h, c)));
}

__global__ void __launch_bounds__(chn::THREADS, 1)
    k_chain_tc(ChainArgs a, const __grid_constant__ CUtensorMap tmZ,
               const __grid_constant__ CUtensorMap tmSfr) {
  using namespace chn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3, h = warp >> 2;
  const int row = q * 32 + lane;
  const bool leader = threadIdx.x == 0;
  const uint32_t bar_mma = sb + OFF_BAR;
  const uint32_t bar_y = bar_mma + 8;
  const uint32_t bar_z = bar_mma + 16;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  const size_t DD = (size_t)D * D;
  const ChainProg g = chain_prog(a, blockIdx.x);
  // Z comes from global memory (TMA) except for the span composite E, whose
  // Z is its own Y (read back from the Y image).
  const bool z_global = !(g.mode == CHAIN_COMPOSE && g.which == 0);
  const bool store_sfr = g.mode == CHAIN_SCAN || g.mode == CHAIN_ADJOINT;  // S_t, or G_t

  if (leader) {
    mbar_init(bar_mma, 1);
    mbar_init(bar_y, 1);
    mbar_init(bar_z, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // Z of step s: matrix index for the tensor map (frame for U, span for H).
  auto z_index = [&](const ChainStep& st) -> int {
    return g.mode == CHAIN_PREFIX ? g.bh * a.nseg + st.t : g.bh * a.T + st.t;
  };
  auto fetch_z = [&](int zi) {
    mbar_arrive_expect_tx(bar_z, kImageBytes);
#pragma unroll
    for (int b = 0; b < 4; ++b) tma_load_3d(sb + OFF_Z + b * ATOM, &tmZ, bar_z, 32 * b, 0, zi);
  };
  int nz = 0, ny = 0, nstore = 0;  // copies issued (leader)
  if (leader && g.n > 0) {
    chain_fetch_y(sb + OFF_Y, chain_step_at(a, g, 0).Y, bar_y);
    ++ny;
    if (z_global) {
      fetch_z(z_index(chain_step_at(a, g, 0)));
      ++nz;
    }
  }

  float x[64];
  load_init_slice(g.init, g.init_hilo, row, h, x);
  float gprod = 1.f;
  // Tile states to store (hi/lo pairs, by TMA): a scan stores each frame's
  // state (the tile at step s holds the state after frame t_{s-1}); the prefix
  // stores each span's start state (the tile at step s holds S_start(s)).
  const bool store_sst = g.mode == CHAIN_PREFIX && a.sst_hilo;
  int tprev = -1;
  auto store_tile = [&](int pair) {
    tma_store_3d(&tmSfr, sb + OFF_XH, 0, 0, 2 * pair);
    tma_store_3d(&tmSfr, sb + OFF_XH + ATOM, 64, 0, 2 * pair);
    tma_store_3d(&tmSfr, sb + OFF_XL, 0, 0, 2 * pair + 1);
    tma_store_3d(&tmSfr, sb + OFF_XL + ATOM, 64, 0, 2 * pair + 1);
    bulk_commit();
    ++nstore;
  };

  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, true);
  for (int s = 0; s < g.n; ++s) {
    const ChainStep st = chain_step_at(a, g, s);
    if (g.mode == CHAIN_PREFIX && !store_sst)
      store_row_f32(a.Sst + ((size_t)g.bh * a.nseg + s) * DD + (size_t)row * D + h * 64, x);
    // A reset (zero state entering this step) is applied in the update below
    // (x <- Z), so the tile still carries the previous frame's state to store.
    // The X tile is free once the previous state store has read it.
    if (leader && nstore > 0) bulk_wait_read0();
    __syncthreads();
    chain_store_x(x, smem + OFF_XH, smem + OFF_XL, row, h);
    fence_proxy_async();
    mbar_wait(bar_y, (uint32_t)s & 1, abort_flag, &g_tc_status, 22);
    float z[64];
    if (!z_global) {
      // Z = Y: this row's slice of the image (hi + lo), read before the buffer is refilled
      const uint8_t* yi = smem + OFF_Y;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 hi = *(const uint4*)(yi + tile_off(row, h, c));
        const uint4 lo = *(const uint4*)(yi + 2 * ATOM + tile_off(row, h, c));
        const uint32_t hw[4] = {hi.x, hi.y, hi.z, hi.w}, lw[4] = {lo.x, lo.y, lo.z, lo.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fh = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hw[e]));
          const float2 fl = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lw[e]));
          z[8 * c + 2 * e] = fh.x + fl.x;
          z[8 * c + 2 * e + 1] = fh.y + fl.y;
        }
      }
    }
    if (__syncthreads_or(*abort_flag != 0)) break;  // one decision for the CTA
    if (leader) {
      if (store_sfr && tprev >= 0) store_tile(g.bh * a.T + tprev);  // S after frame tprev
      if (store_sst) store_tile(g.bh * a.nseg + s);                  // S_start(s)
      tc_fence_after();
      const uint32_t yh = sb + OFF_Y, yl = yh + 2 * ATOM;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t xo = (kk >> 2) * ATOM + (kk & 3) * 32;
        const uint64_t dxh = smem_desc_sw128(sb + OFF_XH + xo, 16, 1024);
        const uint64_t dxl = smem_desc_sw128(sb + OFF_XL + xo, 16, 1024);
        const uint64_t dyh = smem_desc_sw128(yh + kk * 2048, ATOM, 1024);
        const uint64_t dyl = smem_desc_sw128(yl + kk * 2048, ATOM, 1024);
        mma_bf16(tmem, dxh, dyh, idesc, kk > 0 ? 1u : 0u);
        mma_bf16(tmem, dxl, dyh, idesc, 1u);
        mma_bf16(tmem, dxh, dyl, idesc, 1u);
      }
      mma_commit(bar_mma);
    }
    // On a timeout the flag is set; the step finishes on stale values and
    // every thread leaves at the next barrier.
    mbar_wait(bar_mma, (uint32_t)s & 1, abort_flag, &g_tc_status, 21);
    tc_fence_after();
    if (leader && s + 1 < g.n) {  // the Y buffer is free: next step's Y
      chain_fetch_y(sb + OFF_Y, chain_step_at(a, g, s + 1).Y, bar_y);
      ++ny;
    }
    if (z_global) {
      mbar_wait(bar_z, (uint32_t)s & 1, abort_flag, &g_tc_status, 24);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        // columns 64h + 4c .. +3 sit in box (2h + c/8), 16-byte chunk c % 8
        const int box = 2 * h + (c >> 3), ch = c & 7;
        const float4 f = *(const float4*)(smem + OFF_Z + box * ATOM + row * 128 + ((ch ^ (row & 7)) << 4));
        z[4 * c] = f.x; z[4 * c + 1] = f.y; z[4 * c + 2] = f.z; z[4 * c + 3] = f.w;
      }
    }
#pragma unroll
    for (int c0 = 0; c0 < 64; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + h * 64 + c0, r);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c)
        x[c0 + c] = st.reset ? z[c0 + c]
                             : st.alpha * (x[c0 + c] - __uint_as_float(r[c])) + z[c0 + c];
    }
    tc_fence_before();
    if (z_global) {
      // every thread has read Z: fetch the next step's
      __syncthreads();
      if (leader && s + 1 < g.n) {
        fetch_z(z_index(chain_step_at(a, g, s + 1)));
        ++nz;
      }
    }
    if (g.mode == CHAIN_COMPOSE) gprod *= a.gamma[(size_t)g.bh * a.T + st.t];
    if (g.mode == CHAIN_ADJOINT) tprev = st.t;
    if (g.mode == CHAIN_SCAN) {
      tprev = st.t;
      if (g.j0 + s == a.T - 1 && a.state_out)
        store_row_f32(a.state_out + (size_t)g.bh * DD + (size_t)row * D + h * 64, x);
    }
  }
  // the last state of a scan chain (or the last span start of the prefix):
  // through the X tile to its hi/lo store
  if ((store_sfr && tprev >= 0) || store_sst) {
    if (leader && nstore > 0) bulk_wait_read0();
    __syncthreads();
    if (!*abort_flag) {
      chain_store_x(x, smem + OFF_XH, smem + OFF_XL, row, h);
      fence_proxy_async();
    }
    __syncthreads();
    if (leader && !*abort_flag) store_tile(store_sst ? g.bh * a.nseg + g.n : g.bh * a.T + tprev);
  }
  __syncthreads();
  if (!*abort_flag) {
    const size_t si = (size_t)g.bh * a.nseg + g.p;
    if (g.mode == CHAIN_COMPOSE) {
      if (g.which)
        store_row_f32(a.Hc + si * DD + (size_t)row * D + h * 64, x);
      else if (a.e_image)
        store_row_image((uint8_t*)a.E + si * kImageBytes, x, row, h);
      else
        store_row_f32(a.E + si * DD + (size_t)row * D + h * 64, x);
      if (!g.which && threadIdx.x == 0) a.g[si] = gprod;
    } else if (g.mode == CHAIN_PREFIX && !store_sst) {
      store_row_f32(a.Sst + ((size_t)g.bh * a.nseg + g.n) * DD + (size_t)row * D + h * 64, x);
    }
  }
  // Drain (bounded): copies in flight land before teardown.
  if (leader) {
    if (nstore > 0) bulk_wait0();
    if (ny > 0) mbar_wait(bar_y, (uint32_t)(ny - 1) & 1, abort_flag, &g_tc_status, 23);
    if (nz > 0) mbar_wait(bar_z, (uint32_t)(nz - 1) & 1, abort_flag, &g_tc_status, 25);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// fp32 matrix -> operand image; one CTA of 256 threads per matrix.
// An image of a D x D matrix (D = 64 or 128): hi = D/64 blocks of
// [D rows][128 B] (block b holds columns 64b..64b+63), then lo likewise.
__global__ void __launch_bounds__(256) k_to_image(const float* __restrict__ src, uint8_t* __restrict__ dst,
                                                  int D) {
  const float* m = src + (size_t)blockIdx.x * D * D;
  uint8_t* img = dst + (size_t)blockIdx.x * D * D * 4;
  const int cpr = D / 8;  // 16-byte chunks per row
  for (int cid = threadIdx.x; cid < D * cpr; cid += 256) {
    const int k = cid / cpr, nc = cid % cpr;
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = m[k * D + nc * 8 + e];
    const int off = (nc >> 3) * D * 128 + k * 128 + (((nc & 7) ^ (k & 7)) << 4);
    split_chunk(v, (uint4*)(img + off), (uint4*)(img + D * D * 2 + off));
  }
}

cudaError_t tc_to_image(const float* src, void* dst, long long n, int D, cudaStream_t st) {
  k_to_image<<<(unsigned)n, 256, 0, st>>>(src, (uint8_t*)dst, D);
  count_launch();
  return cudaGetLastError();
}

// ============================================================================
// Replay fused with the readout (steps a5 + a6), D = 128.
//
// One CTA takes one chain of CHAIN_SCAN (a span of frames, or a reset block)
// and, frame by frame, first advances the state on tensor cores
//     P = S_{f-1} A_t (3 bf16 products),  S_f = gamma_t (S_{f-1} - P) + U_t
// then streams the frame's Q tiles through
//     O_tile = Q_tile S_f^T = Q_tile S_hi^T + Q_tile S_lo^T.
// The bf16 (hi, lo) state tile in shared memory is at once the A operand of
// the next state step and the B operand of this frame's readout, so S_t never
// goes to HBM. While the readout of frame f streams, the next state step's
// MMA already runs; the state warps write S_{f+1} into the tile as soon as the
// last readout MMA of frame f has drained.
// Roles: warp 0 TMA producer of Q tiles; warp 1 MMA issuer; warps 2-9 hold
// the state (row 32 (w % 4) + lane, columns 64 ((w - 2) / 4) ..) and run the
// readout epilogue (token row 32 (w % 4) + lane of the tile, same columns),
// writing O straight to global memory.
// ============================================================================
namespace sro {
constexpr int D = 128;
constexpr int TOK = 128;
constexpr int NQ = 3;
constexpr int BOX = TOK * 128;          // [128 rows][64 channels] bf16: 16 KiB
constexpr int QT = 2 * BOX;
constexpr int OFF_Q = 0;
constexpr int OFF_X = OFF_Q + NQ * QT;  // state tile: hi (2 atoms) then lo (2 atoms)
constexpr int OFF_Y = OFF_X + 4 * BOX;  // A_t operand image
constexpr int OFF_BAR = OFF_Y + kImageBytes;
constexpr int NBAR = 2 * NQ + 4 + 4 + 1;  // q_full, q_empty, y_full, x_full, p_full, r_done, acc f/e x2, fin
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM = OFF_MISC + 16 + 1024;
constexpr int THREADS = 320;
constexpr uint32_t TMEM_COLS = 512;    // two readout accumulators + the state product
constexpr uint32_t P_COL = 256;
}  // namespace sro

__global__ void __launch_bounds__(sro::THREADS, 1)
    k_scan_readout_tc(ChainArgs a, const __grid_constant__ CUtensorMap tmQ,
                      __nv_bfloat16* __restrict__ out, int S, int nchains) {
  using namespace sro;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_qf = sb + OFF_BAR;
  const uint32_t bar_qe = bar_qf + 8 * NQ;
  const uint32_t bar_yf = bar_qe + 8 * NQ;
  const uint32_t bar_xf = bar_yf + 8;
  const uint32_t bar_pf = bar_xf + 8;
  const uint32_t bar_rd = bar_pf + 8;
  const uint32_t bar_accf = bar_rd + 8;
  const uint32_t bar_acce = bar_accf + 16;
  const uint32_t bar_fin = bar_acce + 16;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  const size_t DD = (size_t)D * D;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NQ; ++s) {
      mbar_init(bar_qf + 8 * s, 1);
      mbar_init(bar_qe + 8 * s, 1);
    }
    mbar_init(bar_yf, 1);
    mbar_init(bar_xf, 8);
    mbar_init(bar_pf, 1);
    mbar_init(bar_rd, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf + 8 * b, 1);
      mbar_init(bar_acce + 8 * b, 8);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int ntile = (S + TOK - 1) / TOK;

  if (warp == 0) {
    // ---- Q tiles of every frame of every chain, in order ----
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int c = blockIdx.x; c < nchains && ok; c += gridDim.x) {
        const ChainProg pg = chain_prog(a, c);
        for (int f = 0; f < pg.n && ok; ++f) {
          const int n = pg.bh * a.T + frame_at(pg.j0 + f, a.T, a.reverse);
          for (int tl = 0; tl < ntile; ++tl, ++g) {
            const int s = g % NQ;
            const uint32_t u = (uint32_t)(g / NQ);
            ok = mbar_wait(bar_qe + 8 * s, (u & 1) ^ 1, abort_flag, &g_tc_status, 31);
            if (!ok) break;
            const uint32_t qd = sb + OFF_Q + s * QT;
            mbar_arrive_expect_tx(bar_qf + 8 * s, QT);
            tma_load_3d(qd, &tmQ, bar_qf + 8 * s, 0, tl * TOK, n);
            tma_load_3d(qd + BOX, &tmQ, bar_qf + 8 * s, 64, tl * TOK, n);
          }
        }
      }
      for (int gg = (g > NQ ? g - NQ : 0); gg < g; ++gg)
        mbar_wait(bar_qf + 8 * (gg % NQ), (uint32_t)(gg / NQ) & 1, abort_flag, &g_tc_status, 32);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer: state step, then the frame's readout tiles ----
    if (lane == 0) {
      constexpr uint32_t id_chain = idesc_bf16_f32(128, 128, false, true);
      constexpr uint32_t id_read = idesc_bf16_f32(128, 128, false, false);
      const uint32_t xh = sb + OFF_X, xl = sb + OFF_X + 2 * BOX;
      int cidx = 0, xidx = 0, g = 0;
      bool ok = true;
      auto chain_mma = [&]() {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t xo = (kk >> 2) * BOX + (kk & 3) * 32;
          const uint64_t dxh = smem_desc_sw128(xh + xo, 16, 1024);
          const uint64_t dxl = smem_desc_sw128(xl + xo, 16, 1024);
          const uint64_t dyh = smem_desc_sw128(sb + OFF_Y + kk * 2048, BOX, 1024);
          const uint64_t dyl = smem_desc_sw128(sb + OFF_Y + 2 * BOX + kk * 2048, BOX, 1024);
          mma_bf16(tmem + P_COL, dxh, dyh, id_chain, kk > 0 ? 1u : 0u);
          mma_bf16(tmem + P_COL, dxl, dyh, id_chain, 1u);
          mma_bf16(tmem + P_COL, dxh, dyl, id_chain, 1u);
        }
        mma_commit(bar_pf);
      };
      for (int c = blockIdx.x; c < nchains && ok; c += gridDim.x) {
        const ChainProg pg = chain_prog(a, c);
        // S_init in the tile -> first state step
        ok = mbar_wait(bar_xf, (uint32_t)(xidx++) & 1, abort_flag, &g_tc_status, 33);
        if (!ok) break;
        ok = mbar_wait(bar_yf, (uint32_t)(cidx++) & 1, abort_flag, &g_tc_status, 34);
        if (!ok) break;
        tc_fence_after();
        chain_mma();
        for (int f = 0; f < pg.n && ok; ++f) {
          ok = mbar_wait(bar_xf, (uint32_t)(xidx++) & 1, abort_flag, &g_tc_status, 35);  // S_f
          if (!ok) break;
          tc_fence_after();
          if (f + 1 < pg.n) {
            ok = mbar_wait(bar_yf, (uint32_t)(cidx++) & 1, abort_flag, &g_tc_status, 36);
            if (!ok) break;
            tc_fence_after();
            chain_mma();
          }
          for (int tl = 0; tl < ntile; ++tl, ++g) {
            const int s = g % NQ;
            const uint32_t u = (uint32_t)(g / NQ);
            const int b = g & 1;
            const uint32_t ub = (uint32_t)(g >> 1);
            ok = mbar_wait(bar_acce + 8 * b, (ub & 1) ^ 1, abort_flag, &g_tc_status, 37);
            if (!ok) break;
            ok = mbar_wait(bar_qf + 8 * s, u & 1, abort_flag, &g_tc_status, 38);
            if (!ok) break;
            tc_fence_after();
            const uint32_t qa = sb + OFF_Q + s * QT;
            const uint32_t d = tmem + b * 128;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * BOX + (kk & 3) * 32;
              const uint64_t dq = smem_desc_sw128(qa + off, 16, 1024);
              const uint64_t dh = smem_desc_sw128(xh + off, 16, 1024);
              const uint64_t dl = smem_desc_sw128(xl + off, 16, 1024);
              mma_bf16(d, dq, dh, id_read, kk > 0 ? 1u : 0u);
              mma_bf16(d, dq, dl, id_read, 1u);
            }
            mma_commit(bar_qe + 8 * s);
            mma_commit(bar_accf + 8 * b);
          }
          mma_commit(bar_rd);
        }
      }
      mma_commit(bar_fin);
      mbar_wait(bar_fin, 0, abort_flag, &g_tc_status, 39);
    }
    __syncwarp();
  } else {
    // ---- state + readout epilogue (256 threads) ----
    const int q = warp & 3, h = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const bool leader = threadIdx.x == 64;
    uint8_t* xtile = smem + OFF_X;
    int pidx = 0, ridx = 0, g = 0, fetched = 0;
    float x[64];
    auto fetch_y = [&](const void* src) {
      if (leader) {
        chain_fetch_y(sb + OFF_Y, src, bar_yf);
        ++fetched;
      }
    };
    auto write_x = [&]() {
      chain_store_x(x, xtile, xtile + 2 * BOX, row, h);
      fence_proxy_async();
      tc_fence_before();
      warp_arrive(bar_xf);
    };
    for (int c = blockIdx.x; c < nchains; c += gridDim.x) {
      const ChainProg pg = chain_prog(a, c);
      if (*abort_flag) break;
      // the previous readout (if any) has drained the tile
      if (ridx > 0) mbar_wait(bar_rd, (uint32_t)(ridx - 1) & 1, abort_flag, &g_tc_status, 40);
      load_init_slice(pg.init, pg.init_hilo, row, h, x);
      fetch_y(chain_step_at(a, pg, 0).Y);
      write_x();
      for (int f = 0; f < pg.n; ++f) {
        const ChainStep st = chain_step_at(a, pg, f);
        const int n = pg.bh * a.T + st.t;
        float z[64];
        {
          const float* zr = st.Z + (size_t)row * D + h * 64;
#pragma unroll
          for (int cc = 0; cc < 64; cc += 4) {
            const float4 v = __ldg((const float4*)(zr + cc));
            z[cc] = v.x; z[cc + 1] = v.y; z[cc + 2] = v.z; z[cc + 3] = v.w;
          }
        }
        mbar_wait(bar_pf, (uint32_t)(pidx++) & 1, abort_flag, &g_tc_status, 41);
        tc_fence_after();
        if (f + 1 < pg.n) fetch_y(chain_step_at(a, pg, f + 1).Y);  // Y buffer is free again
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + P_COL + h * 64 + c0, r);
          tmem_wait_ld();
#pragma unroll
          for (int cc = 0; cc < 32; ++cc)
            x[c0 + cc] = st.alpha * (x[c0 + cc] - __uint_as_float(r[cc])) + z[c0 + cc];
        }
        if (ridx > 0) mbar_wait(bar_rd, (uint32_t)(ridx - 1) & 1, abort_flag, &g_tc_status, 42);
        write_x();  // S_f: readout B operand and the next step's A operand
        if (pg.j0 + f == a.T - 1 && a.state_out)
          store_row_f32(a.state_out + (size_t)pg.bh * DD + (size_t)row * D + h * 64, x);
        // readout epilogue of frame f
        for (int tl = 0; tl < ntile; ++tl, ++g) {
          const int b = g & 1;
          const uint32_t ub = (uint32_t)(g >> 1);
          mbar_wait(bar_accf + 8 * b, ub & 1, abort_flag, &g_tc_status, 43);
          tc_fence_after();
          const int tok = tl * TOK + row;
          __nv_bfloat16* orow = out + ((size_t)n * S + tok) * D + h * 64;
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + b * 128 + h * 64 + c0, r);
            tmem_wait_ld();
            if (tok < S) {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                *(uint4*)(orow + c0 + 8 * j) = make_uint4(
                    pack_bf16x2(__uint_as_float(r[8 * j]), __uint_as_float(r[8 * j + 1])),
                    pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3])),
                    pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5])),
                    pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7])));
            }
          }
          tc_fence_before();
          warp_arrive(bar_acce + 8 * b);
        }
        ++ridx;
      }
    }
    // drain: the last Y copy has landed (its chain MMA normally waited on it)
    if (leader && fetched > 0)
      mbar_wait(bar_yf, (uint32_t)(fetched - 1) & 1, abort_flag, &g_tc_status, 44);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

bool tc_scan_readout_supported(int D) { return D == 128; }

cudaError_t tc_scan_readout(const ChainArgs& a, int nchains, const void* q, void* out, int S,
                            cudaStream_t st) {
  if (a.D != 128 || !a.y_image) return cudaErrorNotSupported;
  CUtensorMap mq;
  const long long N = (long long)a.heads * a.T;
  cudaError_t e = make_map_bf16_3d(&mq, q, 128, S, N, 64, sro::TOK);
  if (e != cudaSuccess) return e;
  static DeviceOnce attr_once;
  const cudaError_t attr_status = once_per_device(attr_once, [&]() -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(k_scan_readout_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             sro::SMEM);
    return e;
  });
  if (attr_status != cudaSuccess) return attr_status;
  const int grid = nchains < num_sms() ? nchains : num_sms();
  k_scan_readout_tc<<<grid, sro::THREADS, sro::SMEM, st>>>(a, mq, (__nv_bfloat16*)out, S, nchains);
  count_launch();
  return cudaGetLastError();
}

bool tc_chain_supported(int D) { return D == 128 || D == 64; }

// 3-D fp32 tensor of D x D matrices, box {32 columns, 128 rows}, 128-byte swizzle.
static cudaError_t make_map_f32_mats(CUtensorMap* m, const void* base, uint64_t n) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {128, 128, n};
  cuuint64_t strides[2] = {128 * 4, 128 * 128 * 4};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

static cudaError_t tc_chain128(const ChainArgs& a, int nchains, cudaStream_t st) {
  if (a.D != 128 || !a.y_image) return cudaErrorNotSupported;
  if (a.mode == CHAIN_SCAN && !a.sfr_hilo) return cudaErrorNotSupported;
  static DeviceOnce attr_once;
  const cudaError_t attr_status = once_per_device(attr_once, [&]() -> cudaError_t {
    cudaError_t e =
        cudaFuncSetAttribute(k_chain_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, chn::SMEM);
    return e;
  });
  if (attr_status != cudaSuccess) return attr_status;
  const long long frames = (long long)a.heads * a.T;
  CUtensorMap mz, ms;
  cudaError_t e;
  if (a.mode == CHAIN_PREFIX)
    e = make_map_f32_mats(&mz, a.Hc, (uint64_t)a.heads * a.nseg);
  else if (a.mode == CHAIN_ADJOINT)
    e = make_map_f32_mats(&mz, a.Zw, (uint64_t)frames);
  else
    e = make_map_f32_mats(&mz, a.U, (uint64_t)frames);
  if (e != cudaSuccess) return e;
  // stored tile states, bf16 hi/lo pairs: per frame (scan) or per span (prefix)
  if (a.mode == CHAIN_PREFIX && a.sst_hilo)
    e = make_map_bf16_3d(&ms, a.Sst, 128, 128, 2 * (uint64_t)a.heads * a.nseg, 64, 128);
  else
    e = make_map_bf16_3d(&ms,
                         a.mode == CHAIN_SCAN      ? (const void*)a.Sfr
                         : a.mode == CHAIN_ADJOINT ? (const void*)a.Gout
                                                   : (const void*)a.U,
                         128, 128, 2 * frames, 64, 128);
  if (e != cudaSuccess) return e;
  k_chain_tc<<<nchains, chn::THREADS, chn::SMEM, st>>>(a, mz, ms);
  count_launch();
  return cudaGetLastError();
}

// ============================================================================
// Contraction and sequential scan in one launch (steps a2 and a5 side by
// side), D = 128.
//
// The contraction is bound by HBM bandwidth and the sequential chain by the
// latency of its steps, so on one GPU they run together: CTAs [0, nchain)
// each run one chain of the recurrence over the frames of one head, while the
// other CTAs run the contraction over frame-heads in scan order (all heads of
// a frame before the next frame). Each contraction epilogue warp publishes its
// rows of A_t, U_t with a release increment of flags[n]; a chain fetches
// frame-head n's operands once flags[n] reaches 4. The launch is cooperative,
// so every CTA is resident and a chain never waits on a CTA that cannot run;
// every wait is bounded.
//
// Chain CTAs use 16 warps: warp w holds rows 32 (w % 4) .. +31 (its TMEM lane
// quadrant) and columns 32 (w / 4) .. +31 of the fp32 state. Per step one
// thread issues P = X_hi Y_hi + X_lo Y_hi + X_hi Y_lo (as the chain kernel
// above), the warps apply X <- gamma (X - P) + U_t, write X back into the
// operand tile as a bf16 (hi, lo) pair and one thread stores that tile (the
// state after frame t) by TMA for the readout.
// ============================================================================
namespace ovl {
constexpr int THREADS = 512;
constexpr int smem(int contract_smem) { return contract_smem > chn::SMEM ? contract_smem : chn::SMEM; }
constexpr int EPI_WARPS = 4;  // contraction epilogue warps: publishes per frame-head
}  // namespace ovl

// Scan step j of a direction: its frame, whether the state entering it is
// replaced (by state_in when `seed`, else by zeros), whether the state after
// it is the direction's final state, the frame whose A image is Y (-1: zeros)
// and the frame whose gamma is alpha (-1: 1).
struct OvlStep {
  int t, reset, seed, last, yt, at;
};

__device__ __forceinline__ OvlStep ovl_step(const OvlDir& d, int T, int block, int j) {
  OvlStep s;
  if (d.adjoint) {
    const int jf = T - 1 - j;  // forward scan position
    s.t = d.reverse ? T - 1 - jf : jf;
    s.last = 0;
    if (j == 0) {
      s.reset = s.seed = 1;  // G starts from dL/d(state_out)
      s.yt = s.at = -1;
    } else {
      const int tn = d.reverse ? T - 2 - jf : jf + 1;  // next frame in forward order
      s.reset = d.seq_reset && (s.t / block) != (tn / block);
      s.seed = 0;
      s.yt = s.at = tn;
    }
    return s;
  }
  if (d.blocks_asc) {
    const int b = j / block, o = j - b * block;
    const int t1 = min(b * block + block, T);
    s.t = t1 - 1 - o;
    s.reset = o == 0;
    s.seed = o == 0 && t1 == T;  // the block holding frame T-1 comes first in scan order
    s.last = s.t == 0;
  } else {
    s.t = d.reverse ? T - 1 - j : j;
    const int tp = d.reverse ? s.t + 1 : s.t - 1;
    s.reset = j == 0 || (d.seq_reset && (s.t / block) != (tp / block));
    s.seed = j == 0;
    s.last = j == T - 1;
  }
  s.yt = s.at = s.t;
  return s;
}

// Bounded wait until *f >= target (acquire); false on abort or timeout.
__device__ __forceinline__ bool wait_flag_ge(const int* f, int target, volatile int* abort_flag,
                                             int code) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
  if (v >= target) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    if (v >= target) return true;
    if ((it & 15u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > kWaitNs) {
        atomicCAS(&g_tc_status, 0, code);  // the first wait to run out is the cause
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// 32 consecutive fp32 values of a row (16-byte aligned), or zeros.
__device__ __forceinline__ void load_row32(const float* src, float* x) {
  if (!src) {
#pragma unroll
    for (int c = 0; c < 32; ++c) x[c] = 0.f;
    return;
  }
#pragma unroll
  for (int c = 0; c < 32; c += 4) {
    const float4 f = __ldg((const float4*)(src + c));
    x[c] = f.x; x[c + 1] = f.y; x[c + 2] = f.z; x[c + 3] = f.w;
  }
}

// The thread's 32 state values (row `row`, columns 32 cg ..) into the X tile
// as bf16 (hi, lo): atom cg / 2, 16-byte chunks 4 (cg % 2) .. +3.
__device__ __forceinline__ void ovl_store_x(const float* x, uint8_t* xh, uint8_t* xl, int row,
                                            int cg) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 hi, lo;
    split_chunk(x + 8 * i, &hi, &lo);
    const int off = tile_off(row, cg >> 1, 4 * (cg & 1) + i);
    *(uint4*)(xh + off) = hi;
    *(uint4*)(xl + off) = lo;
  }
}

// Chain role of the overlapped launch: chain c = direction c / heads, head c % heads.
__device__ __forceinline__ void ovl_chain_body(const OvlArgs& o, const CUtensorMap& tmZ,
                                               const CUtensorMap& tmS0, const CUtensorMap& tmS1,
                                               int c) {
  using namespace chn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3, cg = warp >> 2;
  const int row = q * 32 + lane;
  const bool leader = threadIdx.x == 0;
  const uint32_t bar_mma = sb + OFF_BAR;
  const uint32_t bar_y = bar_mma + 8;
  const uint32_t bar_z = bar_mma + 16;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  const int di = c / o.heads, bh = c % o.heads;
  const OvlDir d = di ? o.dir[1] : o.dir[0];
  const CUtensorMap* tmS = di ? &tmS1 : &tmS0;
  const int T = o.T;
  const size_t DD = (size_t)D * D;

  if (leader) {
    mbar_init(bar_mma, 1);
    mbar_init(bar_y, 1);
    mbar_init(bar_z, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // operands of the frame at scan step j: wait for its publication, then copy
  int ny = 0, nz = 0, nstore = 0;  // copies issued (leader)
  // Y of a step: the A image of st.yt (zeros when -1), once frame st.t's
  // contraction output is published
  auto fetch_y = [&](const OvlStep& st) -> bool {
    const int n = bh * T + st.t;
    if (!wait_flag_ge(o.flags + n, ovl::EPI_WARPS, abort_flag, 31)) return false;
    asm volatile("fence.proxy.async.global;" ::: "memory");
    chain_fetch_y(sb + OFF_Y,
                  st.yt >= 0 ? o.A + ((size_t)bh * T + st.yt) * kImageBytes : o.zero_img, bar_y);
    ++ny;
    return true;
  };
  auto fetch_z = [&](int t) {
    const int n = bh * T + t;
    mbar_arrive_expect_tx(bar_z, kImageBytes);
#pragma unroll
    for (int b = 0; b < 4; ++b) tma_load_3d(sb + OFF_Z + b * ATOM, &tmZ, bar_z, 32 * b, 0, n);
    ++nz;
  };
  if (leader && T > 0) {
    const OvlStep s0 = ovl_step(d, T, o.block, 0);
    if (fetch_y(s0)) fetch_z(s0.t);
  }

  float x[32];
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, true);
  for (int j = 0; j < T; ++j) {
    const OvlStep st = ovl_step(d, T, o.block, j);
    if (st.reset) {
      // the state entering this step is replaced; the tile must be free first
      if (leader && nstore > 0) bulk_wait_read0();
      __syncthreads();
      const float* init = st.seed && d.state_in ? d.state_in + (size_t)bh * DD : nullptr;
      load_row32(init ? init + (size_t)row * D + 32 * cg : nullptr, x);
      ovl_store_x(x, smem + OFF_XH, smem + OFF_XL, row, cg);
      fence_proxy_async();
    }
    mbar_wait(bar_y, (uint32_t)j & 1, abort_flag, &g_tc_status, 32);
    if (__syncthreads_or(*abort_flag != 0)) break;  // one decision for the CTA
    if (leader) {
      tc_fence_after();
      const uint32_t yh = sb + OFF_Y, yl = yh + 2 * ATOM;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t xo = (kk >> 2) * ATOM + (kk & 3) * 32;
        const uint64_t dxh = smem_desc_sw128(sb + OFF_XH + xo, 16, 1024);
        const uint64_t dxl = smem_desc_sw128(sb + OFF_XL + xo, 16, 1024);
        const uint64_t dyh = smem_desc_sw128(yh + kk * 2048, ATOM, 1024);
        const uint64_t dyl = smem_desc_sw128(yl + kk * 2048, ATOM, 1024);
        mma_bf16(tmem, dxh, dyh, idesc, kk > 0 ? 1u : 0u);
        mma_bf16(tmem, dxl, dyh, idesc, 1u);
        mma_bf16(tmem, dxh, dyl, idesc, 1u);
      }
      mma_commit(bar_mma);
    }
    mbar_wait(bar_mma, (uint32_t)j & 1, abort_flag, &g_tc_status, 33);
    tc_fence_after();
    // the Y buffer is free: the next step's image, once its frame is published
    int tn = -1;
    if (j + 1 < T) {
      const OvlStep sn = ovl_step(d, T, o.block, j + 1);
      tn = sn.t;
      if (leader) fetch_y(sn);
    }
    mbar_wait(bar_z, (uint32_t)j & 1, abort_flag, &g_tc_status, 34);
    if (o.discard && leader) {
      // this frame's A_t image and U_t now sit in shared memory: one more count
      // on its flag tells the contraction CTA that wrote them that their L2
      // lines can go unwritten (it drops them off this chain's critical path)
      asm volatile("red.relaxed.gpu.global.add.s32 [%0], %1;" ::"l"(o.flags + (size_t)bh * T + st.t),
                   "r"(1)
                   : "memory");
    }
    {
      const float alpha = st.at >= 0 ? o.gamma[(size_t)bh * T + st.at] : 1.f;
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + 32 * cg, r);
      tmem_wait_ld();
      const uint8_t* zb = smem + OFF_Z + cg * ATOM + row * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const float4 z = *(const float4*)(zb + ((ch ^ (row & 7)) << 4));
        x[4 * ch] = alpha * (x[4 * ch] - __uint_as_float(r[4 * ch])) + z.x;
        x[4 * ch + 1] = alpha * (x[4 * ch + 1] - __uint_as_float(r[4 * ch + 1])) + z.y;
        x[4 * ch + 2] = alpha * (x[4 * ch + 2] - __uint_as_float(r[4 * ch + 2])) + z.z;
        x[4 * ch + 3] = alpha * (x[4 * ch + 3] - __uint_as_float(r[4 * ch + 3])) + z.w;
      }
    }
    tc_fence_before();
    // every thread has read Z and P; the previous state store has read the tile
    if (leader && nstore > 0) bulk_wait_read0();
    __syncthreads();
    if (leader && tn >= 0 && !*abort_flag) fetch_z(tn);
    ovl_store_x(x, smem + OFF_XH, smem + OFF_XL, row, cg);
    fence_proxy_async();
    if (st.last && d.state_out) {
      float* so = d.state_out + (size_t)bh * DD + (size_t)row * D + 32 * cg;
#pragma unroll
      for (int c4 = 0; c4 < 32; c4 += 4)
        *(float4*)(so + c4) = make_float4(x[c4], x[c4 + 1], x[c4 + 2], x[c4 + 3]);
    }
    __syncthreads();
    if (leader) {
      // the state after frame t, as a bf16 (hi, lo) pair, for the readout
      const int pair = bh * T + st.t;
      tma_store_3d(tmS, sb + OFF_XH, 0, 0, 2 * pair);
      tma_store_3d(tmS, sb + OFF_XH + ATOM, 64, 0, 2 * pair);
      tma_store_3d(tmS, sb + OFF_XL, 0, 0, 2 * pair + 1);
      tma_store_3d(tmS, sb + OFF_XL + ATOM, 64, 0, 2 * pair + 1);
      bulk_commit();
      ++nstore;
    }
  }
  // Drain (bounded, and not cut short by an abort): copies in flight land
  // before teardown.
  if (leader) {
    volatile int keep_waiting = 0;
    if (nstore > 0) bulk_wait0();
    if (ny > 0) mbar_wait(bar_y, (uint32_t)(ny - 1) & 1, &keep_waiting, &g_tc_status, 35);
    if (nz > 0) mbar_wait(bar_z, (uint32_t)(nz - 1) & 1, &keep_waiting, &g_tc_status, 36);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int NST, bool UC = false>
__global__ void __launch_bounds__(ovl::THREADS, 1)
    k_contract_scan_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const float* __restrict__ beta, float* __restrict__ A, float* __restrict__ U,
                       int N, int S, float cA, float cU, ProArgs pro, OvlArgs o, int nchain,
                       const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmS0,
                       const __grid_constant__ CUtensorMap tmS1) {
  if ((int)blockIdx.x < nchain)
    ovl_chain_body(o, tmZ, tmS0, tmS1, blockIdx.x);
  else
    contract_body<NST, UC>(tmK, tmV, beta, A, U, N, S, cA, cU, o.a_image, pro,
                           (int)blockIdx.x - nchain, (int)gridDim.x - nchain, o.heads, o.T,
                           o.contract_rev, o.flags, 1, o.discard);
}

bool tc_overlap_supported(int D) { return D == 128; }
int tc_num_sms() { return num_sms(); }
int tc_overlap_max_chains() { return num_sms() / 4; }

cudaError_t tc_contract_scan(const void* k, const void* v, const float* beta, float* A, float* U,
                             long long N, int S, float cA, float cU, const ProArgs* pro,
                             const OvlArgs& o, void* sfr0, void* sfr1, cudaStream_t st) {
  if (pro && pro->npos * (128 / 4) > ctr::TAB_MAX) return cudaErrorNotSupported;
  const int nchain = o.ndir * o.heads;
  if (o.ndir < 1 || o.ndir > 2 || nchain > tc_overlap_max_chains() ||
      (long long)o.heads * o.T != N)
    return cudaErrorNotSupported;
  ProArgs pa = {};
  if (pro) pa = *pro;
  CUtensorMap mk, mv, mz, ms0, ms1;
  cudaError_t e = make_map_bf16_3d(&mk, k, 128, S, N, 64, ctr::TOK);
  if (e == cudaSuccess) e = make_map_bf16_3d(&mv, v, 128, S, N, 64, ctr::TOK);
  if (e == cudaSuccess) e = make_map_f32_mats(&mz, U, (uint64_t)N);
  if (e == cudaSuccess) e = make_map_bf16_3d(&ms0, sfr0, 128, 128, 2 * (uint64_t)N, 64, 128);
  if (e == cudaSuccess)
    e = make_map_bf16_3d(&ms1, sfr1 ? sfr1 : sfr0, 128, 128, 2 * (uint64_t)N, 64, 128);
  if (e != cudaSuccess) return e;
  constexpr int smem_plain = ovl::smem(ctr::SMEM_PLAIN), smem_pro = ovl::smem(ctr::SMEM_PRO);
  static DeviceOnce attr_once;
  const cudaError_t attr_status = once_per_device(attr_once, [&]() -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(k_contract_scan_tc<ctr::NST_PLAIN>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem_plain);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_contract_scan_tc<ctr::NST_PRO>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem_pro);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_contract_scan_tc<ctr::NST_PRO, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem_pro);
    return e;
  });
  if (attr_status != cudaSuccess) return attr_status;
  long long ncon = num_sms() - nchain;
  if (ncon > N) ncon = N;
  const int grid = nchain + (int)ncon;
  e = cudaMemsetAsync(o.flags, 0, (size_t)N * sizeof(int), st);
  if (e != cudaSuccess) return e;
  const float* beta_a = beta;
  float *A_a = A, *U_a = U;
  int N_a = (int)N, S_a = S, nchain_a = nchain;
  float cA_a = cA, cU_a = cU;
  OvlArgs o_a = o;
  o_a.U = U;
  void* args[] = {&mk, &mv, &beta_a, &A_a, &U_a, &N_a, &S_a, &cA_a, &cU_a,
                  &pa, &o_a, &nchain_a, &mz, &ms0, &ms1};
  // cooperative: every CTA is resident, so the chains' waits on the
  // contraction CTAs always end
  if (pro && pro->ucpe)
    e = cudaLaunchCooperativeKernel((const void*)k_contract_scan_tc<ctr::NST_PRO, true>, dim3(grid),
                                    dim3(ovl::THREADS), args, (size_t)smem_pro, st);
  else if (pro)
    e = cudaLaunchCooperativeKernel((const void*)k_contract_scan_tc<ctr::NST_PRO>, dim3(grid),
                                    dim3(ovl::THREADS), args, (size_t)smem_pro, st);
  else
    e = cudaLaunchCooperativeKernel((const void*)k_contract_scan_tc<ctr::NST_PLAIN>, dim3(grid),
                                    dim3(ovl::THREADS), args, (size_t)smem_plain, st);
  count_launch();
  return e;
}

// ============================================================================
// D = 64 tensor-core kernels.
//
// Contraction: [K^T; V^T] is one M = 128 MN-major operand (the K and V boxes
// of a stage sit next to each other, LBO = one box) against beta*K (N = 64),
// so one 128x64x16 MMA per 16 tokens yields [A_t; U_t] in TMEM rows 0-63 /
// 64-127. Readout: M = 128 tokens, N = 64, one 128-byte swizzle atom wide.
// Chains: the state is 64 x 64; a span's E and H chains share Y = A_t and run
// stacked in one CTA (E in rows 0-63, H in rows 64-127); a scan or prefix chain
// uses rows 0-63 only. Operand images for D = 64: hi [64 rows][128 B] then lo.
// ============================================================================
namespace c64 {
constexpr int D = 64;
constexpr int TOK = 64;
constexpr int NST = 6;
constexpr int BOX = TOK * 128;        // [64 tokens][64 channels] bf16: 8 KiB
constexpr int KV = 2 * BOX;           // K box, then V box: the stacked A operand
constexpr int OFF_KV = 0;
constexpr int OFF_BK = OFF_KV + NST * KV;
constexpr int OFF_BETA = OFF_BK + NST * BOX;
constexpr int OFF_BAR = OFF_BETA + NST * TOK * 4;
constexpr int NBAR = 3 * NST + 5;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM = OFF_MISC + 16 + 1024;
constexpr int NSC = 128;
constexpr int THREADS = 64 + NSC + 128;
constexpr uint32_t TMEM_COLS = 128;
constexpr int IMG = D * D * 4;        // operand image bytes
}  // namespace c64

__global__ void __launch_bounds__(c64::THREADS, 1)
    k_contract64_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const float* __restrict__ beta, float* __restrict__ A, float* __restrict__ U,
                    int N, int S, float cA, float cU, int a_image) {
  using namespace c64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_full = sb + OFF_BAR;
  const uint32_t bar_bk = bar_full + 8 * NST;
  const uint32_t bar_empty = bar_bk + 8 * NST;
  const uint32_t bar_accf = bar_empty + 8 * NST;
  const uint32_t bar_acce = bar_accf + 16;
  const uint32_t bar_fin = bar_acce + 16;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full + 8 * s, 33);
      mbar_init(bar_bk + 8 * s, NSC / 32);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf + 8 * b, 1);
      mbar_init(bar_acce + 8 * b, 4);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int nst_frame = (S + TOK - 1) / TOK;
  const int my_count = (int)blockIdx.x < N ? (N - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp == 0) {
    int g = 0;
    bool ok = true;
    for (int i = 0; i < my_count && ok; ++i) {
      const int n = blockIdx.x + i * gridDim.x;
      for (int st = 0; st < nst_frame; ++st, ++g) {
        const int s = g % NST;
        const uint32_t u = (uint32_t)(g / NST);
        if (lane == 0) ok = mbar_wait(bar_empty + 8 * s, (u & 1) ^ 1, abort_flag, &g_tc_status, 51);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          const uint32_t kd = sb + OFF_KV + s * KV;
          mbar_arrive_expect_tx(bar_full + 8 * s, KV);
          tma_load_3d(kd, &tmK, bar_full + 8 * s, 0, st * TOK, n);
          tma_load_3d(kd + BOX, &tmV, bar_full + 8 * s, 0, st * TOK, n);
        }
        const uint32_t bsa = sb + OFF_BETA + s * TOK * 4;
#pragma unroll
        for (int r = lane; r < TOK; r += 32) {
          const int tok = st * TOK + r;
          const bool in = tok < S;
          cp_async_4(bsa + r * 4, beta + (size_t)n * S + (in ? tok : 0), in ? 4u : 0u);
        }
        cp_async_arrive_noinc(bar_full + 8 * s);
      }
    }
    if (lane == 0) {
      for (int gg = (g > NST ? g - NST : 0); gg < g; ++gg)
        mbar_wait(bar_full + 8 * (gg % NST), (uint32_t)(gg / NST) & 1, abort_flag, &g_tc_status, 52);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 64, true, true);
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_count && ok; ++i) {
        const int b = i & 1;
        const uint32_t ub = (uint32_t)(i >> 1);
        ok = mbar_wait(bar_acce + 8 * b, (ub & 1) ^ 1, abort_flag, &g_tc_status, 53);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + b * 64;
        for (int st = 0; st < nst_frame; ++st, ++g) {
          const int s = g % NST;
          const uint32_t u = (uint32_t)(g / NST);
          ok = mbar_wait(bar_bk + 8 * s, u & 1, abort_flag, &g_tc_status, 54);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kva = sb + OFF_KV + s * KV, ba = sb + OFF_BK + s * BOX;
#pragma unroll
          for (int kk = 0; kk < TOK / 16; ++kk) {
            const uint64_t da = smem_desc_sw128(kva + kk * 2048, BOX, 1024);  // [K^T; V^T]
            const uint64_t db = smem_desc_sw128(ba + kk * 2048, BOX, 1024);
            mma_bf16(d, da, db, idesc, (st > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar_empty + 8 * s);
        }
        if (!ok) break;
        mma_commit(bar_accf + 8 * b);
      }
      mma_commit(bar_fin);
      mbar_wait(bar_fin, 0, abort_flag, &g_tc_status, 55);
    }
    __syncwarp();
  } else if (warp < 2 + NSC / 32) {
    const int t = threadIdx.x - 64;
    int g = 0;
    bool ok = true;
    for (int i = 0; i < my_count && ok; ++i) {
      for (int st = 0; st < nst_frame; ++st, ++g) {
        const int s = g % NST;
        const uint32_t u = (uint32_t)(g / NST);
        ok = mbar_wait(bar_full + 8 * s, u & 1, abort_flag, &g_tc_status, 56);
        if (!ok) break;
        const uint8_t* kt = smem + OFF_KV + s * KV;
        uint8_t* bt = smem + OFF_BK + s * BOX;
        const float* bs = (const float*)(smem + OFF_BETA) + s * TOK;
#pragma unroll
        for (int m = 0; m < (BOX / 16) / NSC; ++m) {
          const int c = t + NSC * m;
          const float bv = bs[c >> 3];
          uint4 x = *(const uint4*)(kt + c * 16);
          uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w[e]));
            w[e] = pack_bf16x2(f.x * bv, f.y * bv);
          }
          *(uint4*)(bt + c * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async();
        warp_arrive(bar_bk + 8 * s);
      }
    }
  } else {
    // TMEM rows 0-63 hold A_t, rows 64-127 U_t
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const bool isA = row < 64;
    const int r = isA ? row : row - 64;
    for (int i = 0; i < my_count; ++i) {
      const int b = i & 1;
      const uint32_t ub = (uint32_t)(i >> 1);
      if (!mbar_wait(bar_accf + 8 * b, ub & 1, abort_flag, &g_tc_status, 57)) break;
      tc_fence_after();
      const int n = blockIdx.x + i * gridDim.x;
      const float sc = isA ? cA : cU;
#pragma unroll
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t rr[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + b * 64 + c0, rr);
        tmem_wait_ld();
        if (isA && a_image) {
          uint8_t* img = (uint8_t*)A + (size_t)n * IMG;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(rr[8 * j + e]) * sc;
            const int off = r * 128 + ((((c0 >> 3) + j) ^ (r & 7)) << 4);
            split_chunk(v, (uint4*)(img + off), (uint4*)(img + D * D * 2 + off));
          }
        } else {
          float* dst = (isA ? A : U) + ((size_t)n * D + r) * D + c0;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *(float4*)(dst + 4 * j) =
                make_float4(__uint_as_float(rr[4 * j]) * sc, __uint_as_float(rr[4 * j + 1]) * sc,
                            __uint_as_float(rr[4 * j + 2]) * sc, __uint_as_float(rr[4 * j + 3]) * sc);
        }
      }
      tc_fence_before();
      warp_arrive(bar_acce + 8 * b);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

namespace r64 {
constexpr int D = 64;
constexpr int TOK = 128;
constexpr int NQ = 4;
constexpr int QBOX = TOK * 128;          // [128 tokens][64 channels] bf16: 16 KiB
constexpr int SBOX = 64 * 128;           // [64 rows][64] bf16: 8 KiB
constexpr int OFF_Q = 0;
constexpr int OFF_S = OFF_Q + NQ * QBOX; // S hi, then S lo
constexpr int OFF_O = OFF_S + 2 * SBOX;  // output staging: one box
constexpr int OFF_BAR = OFF_O + QBOX;
constexpr int NBAR = 2 * NQ + 2 + 4 + 1;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM = OFF_MISC + 16 + 1024;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 128;
}  // namespace r64

__global__ void __launch_bounds__(r64::THREADS, 1)
    k_readout64_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmS,
                   const __grid_constant__ CUtensorMap tmO, int N, int S, int parts) {
  using namespace r64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_qf = sb + OFF_BAR;
  const uint32_t bar_qe = bar_qf + 8 * NQ;
  const uint32_t bar_sf = bar_qe + 8 * NQ;
  const uint32_t bar_se = bar_sf + 8;
  const uint32_t bar_accf = bar_se + 8;
  const uint32_t bar_acce = bar_accf + 16;
  const uint32_t bar_fin = bar_acce + 16;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  if (threadIdx.x == 0) {
    for (int s = 0; s < NQ; ++s) {
      mbar_init(bar_qf + 8 * s, 1);
      mbar_init(bar_qe + 8 * s, 1);
    }
    mbar_init(bar_sf, 1);
    mbar_init(bar_se, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf + 8 * b, 1);
      mbar_init(bar_acce + 8 * b, 4);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int ntile = (S + TOK - 1) / TOK;
  // Work units: each frame-head's tiles in kParts contiguous parts (outputs are
  // per token, so parts need no reduction); finer units even out the rounds.
  const int kParts = parts;
  const int NU = N * kParts;
  const int my_count = (int)blockIdx.x < NU ? (NU - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp == 0) {
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_count && ok; ++i) {
        const int unit = blockIdx.x + i * gridDim.x;
        const int n = unit / kParts, part = unit % kParts;
        const int tl0 = part * ntile / kParts, tl1 = (part + 1) * ntile / kParts;
        (void)n;
                ok = mbar_wait(bar_se, ((uint32_t)i & 1) ^ 1, abort_flag, &g_tc_status, 61);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_sf, 2 * SBOX);
        tma_load_3d(sb + OFF_S, &tmS, bar_sf, 0, 0, 2 * n);
        tma_load_3d(sb + OFF_S + SBOX, &tmS, bar_sf, 0, 0, 2 * n + 1);
        for (int tl = tl0; tl < tl1; ++tl, ++g) {
          const int s = g % NQ;
          const uint32_t u = (uint32_t)(g / NQ);
          ok = mbar_wait(bar_qe + 8 * s, (u & 1) ^ 1, abort_flag, &g_tc_status, 62);
          if (!ok) break;
          mbar_arrive_expect_tx(bar_qf + 8 * s, QBOX);
          tma_load_3d(sb + OFF_Q + s * QBOX, &tmQ, bar_qf + 8 * s, 0, tl * TOK, n);
        }
      }
      for (int gg = (g > NQ ? g - NQ : 0); gg < g; ++gg)
        mbar_wait(bar_qf + 8 * (gg % NQ), (uint32_t)(gg / NQ) & 1, abort_flag, &g_tc_status, 63);
      if (my_count > 0) mbar_wait(bar_sf, (uint32_t)(my_count - 1) & 1, abort_flag, &g_tc_status, 64);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 64, false, false);
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_count && ok; ++i) {
        const int unit = blockIdx.x + i * gridDim.x;
        const int n = unit / kParts, part = unit % kParts;
        const int tl0 = part * ntile / kParts, tl1 = (part + 1) * ntile / kParts;
        (void)n;
        ok = mbar_wait(bar_sf, (uint32_t)i & 1, abort_flag, &g_tc_status, 65);
        if (!ok) break;
        tc_fence_after();
        for (int tl = tl0; tl < tl1; ++tl, ++g) {
          const int s = g % NQ;
          const uint32_t u = (uint32_t)(g / NQ);
          const int b = g & 1;
          const uint32_t ub = (uint32_t)(g >> 1);
          ok = mbar_wait(bar_acce + 8 * b, (ub & 1) ^ 1, abort_flag, &g_tc_status, 66);
          if (!ok) break;
          ok = mbar_wait(bar_qf + 8 * s, u & 1, abort_flag, &g_tc_status, 67);
          if (!ok) break;
          tc_fence_after();
          const uint32_t qa = sb + OFF_Q + s * QBOX;
          const uint32_t d = tmem + b * 64;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t dq = smem_desc_sw128(qa + kk * 32, 16, 1024);
            const uint64_t dh = smem_desc_sw128(sb + OFF_S + kk * 32, 16, 1024);
            const uint64_t dl = smem_desc_sw128(sb + OFF_S + SBOX + kk * 32, 16, 1024);
            mma_bf16(d, dq, dh, idesc, kk > 0 ? 1u : 0u);
            mma_bf16(d, dq, dl, idesc, 1u);
          }
          mma_commit(bar_qe + 8 * s);
          mma_commit(bar_accf + 8 * b);
        }
        if (!ok) break;
        mma_commit(bar_se);
      }
      mma_commit(bar_fin);
      mbar_wait(bar_fin, 0, abort_flag, &g_tc_status, 68);
    }
    __syncwarp();
  } else {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int et = threadIdx.x - 64;
    uint8_t* ost = smem + OFF_O;
    int g = 0;
    bool ok = true;
    for (int i = 0; i < my_count && ok; ++i) {
      const int unit = blockIdx.x + i * gridDim.x;
      const int n = unit / kParts, part = unit % kParts;
      const int tl0 = part * ntile / kParts, tl1 = (part + 1) * ntile / kParts;
      (void)n;
            for (int tl = tl0; tl < tl1; ++tl, ++g) {
        const int b = g & 1;
        const uint32_t ub = (uint32_t)(g >> 1);
        mbar_wait(bar_accf + 8 * b, ub & 1, abort_flag, &g_tc_status, 69);
        tc_fence_after();
        if (et == 0) bulk_wait_read0();
        if (named_bar_or(1, 128, *abort_flag != 0)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 32) {
          uint32_t rr[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + b * 64 + c0, rr);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *(uint4*)(ost + row * 128 + ((((c0 >> 3) + j) ^ (row & 7)) << 4)) = make_uint4(
                pack_bf16x2(__uint_as_float(rr[8 * j]), __uint_as_float(rr[8 * j + 1])),
                pack_bf16x2(__uint_as_float(rr[8 * j + 2]), __uint_as_float(rr[8 * j + 3])),
                pack_bf16x2(__uint_as_float(rr[8 * j + 4]), __uint_as_float(rr[8 * j + 5])),
                pack_bf16x2(__uint_as_float(rr[8 * j + 6]), __uint_as_float(rr[8 * j + 7])));
        }
        tc_fence_before();
        warp_arrive(bar_acce + 8 * b);
        fence_proxy_async();
        named_bar_sync(1, 128);
        if (et == 0) {
          tma_store_3d(&tmO, sb + OFF_O, 0, tl * TOK, n);
          bulk_commit();
        }
      }
    }
    if (et == 0) bulk_wait0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

namespace h64 {
constexpr int D = 64;
constexpr int XT = 128 * 128;            // X tile: 128 rows x 64 bf16 (one atom): 16 KiB
constexpr int OFF_XH = 0;
constexpr int OFF_XL = OFF_XH + XT;
constexpr int OFF_Y = OFF_XL + XT;       // operand image (hi 8 KiB, lo 8 KiB)
constexpr int OFF_Z = OFF_Y + c64::IMG;  // Z fp32: 2 boxes of [64 rows][32 fp32]
constexpr int OFF_BAR = OFF_Z + c64::IMG;
constexpr int OFF_MISC = OFF_BAR + 32;
constexpr int SMEM = OFF_MISC + 16 + 1024;
constexpr int THREADS = 256;
constexpr uint32_t TMEM_COLS = 64;
}  // namespace h64

// Rows 0-63 run the chain; for a span composite they run E and rows 64-127 run
// H of the same span (same Y). Each thread: row 32 (w % 4) + lane, columns
// 32 (w / 4) .. +31.
__global__ void __launch_bounds__(h64::THREADS)
    k_chain64_tc(ChainArgs a, const __grid_constant__ CUtensorMap tmZ,
                 const __grid_constant__ CUtensorMap tmSt) {
  using namespace h64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3, h = warp >> 2;
  const int row = q * 32 + lane;
  const bool top = row < 64;
  const int r = top ? row : row - 64;
  const bool leader = threadIdx.x == 0;
  const uint32_t bar_mma = sb + OFF_BAR;
  const uint32_t bar_y = bar_mma + 8;
  const uint32_t bar_z = bar_mma + 16;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  const size_t DD = (size_t)D * D;
  const bool compose = a.mode == CHAIN_COMPOSE;
  // one CTA per span for the composites: E (rows 0-63) and H (rows 64-127)
  ChainProg g = chain_prog(a, blockIdx.x);
  const bool active = compose || top;                 // rows that carry a chain
  const bool zy = compose && top;                     // E rows: Z = Y
  const bool store_sfr = g.mode == CHAIN_SCAN;
  const bool store_sst = g.mode == CHAIN_PREFIX && a.sst_hilo;
  if (leader) {
    mbar_init(bar_mma, 1);
    mbar_init(bar_y, 1);
    mbar_init(bar_z, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  auto z_index = [&](const ChainStep& st) -> int {
    return g.mode == CHAIN_PREFIX ? g.bh * a.nseg + st.t : g.bh * a.T + st.t;
  };
  auto fetch_y = [&](const void* src) {
    mbar_arrive_expect_tx(bar_y, c64::IMG);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            sb + OFF_Y),
        "l"(src), "r"((uint32_t)c64::IMG), "r"(bar_y)
        : "memory");
  };
  auto fetch_z = [&](int zi) {
    mbar_arrive_expect_tx(bar_z, c64::IMG);
    tma_load_3d(sb + OFF_Z, &tmZ, bar_z, 0, 0, zi);
    tma_load_3d(sb + OFF_Z + 64 * 128, &tmZ, bar_z, 32, 0, zi);
  };
  int nz = 0, ny = 0, nstore = 0;
  if (leader && g.n > 0) {
    fetch_y(chain_step_at(a, g, 0).Y);
    ++ny;
    fetch_z(z_index(chain_step_at(a, g, 0)));
    ++nz;
  }
  float x[32];
  {
    const bool has_init = top && g.init;
    if (!has_init) {
#pragma unroll
      for (int c = 0; c < 32; ++c) x[c] = 0.f;
    } else if (g.init_hilo) {
      const __nv_bfloat16* hi = (const __nv_bfloat16*)g.init + (size_t)r * D + h * 32;
      const __nv_bfloat16* lo = hi + DD;
#pragma unroll
      for (int c = 0; c < 32; ++c) x[c] = __bfloat162float(hi[c]) + __bfloat162float(lo[c]);
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) x[c] = g.init[(size_t)r * D + h * 32 + c];
    }
  }
  float gprod = 1.f;
  int tprev = -1;
  auto store_tile = [&](int pair) {  // rows 0-63 of the X tile: S hi/lo, one [64][64] box each
    tma_store_3d(&tmSt, sb + OFF_XH, 0, 0, 2 * pair);
    tma_store_3d(&tmSt, sb + OFF_XL, 0, 0, 2 * pair + 1);
    bulk_commit();
    ++nstore;
  };
  auto write_x = [&]() {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint4 hi, lo;
      split_chunk(x + 8 * c, &hi, &lo);
      const int off = row * 128 + (((4 * h + c) ^ (row & 7)) << 4);
      *(uint4*)(smem + OFF_XH + off) = hi;
      *(uint4*)(smem + OFF_XL + off) = lo;
    }
  };
  constexpr uint32_t idesc = idesc_bf16_f32(128, 64, false, true);
  for (int s = 0; s < g.n; ++s) {
    const ChainStep st = chain_step_at(a, g, s);
    if (g.mode == CHAIN_PREFIX && !store_sst && top)
      for (int c = 0; c < 32; ++c) a.Sst[((size_t)g.bh * a.nseg + s) * DD + (size_t)r * D + h * 32 + c] = x[c];
    if (leader && nstore > 0) bulk_wait_read0();
    __syncthreads();
    write_x();
    fence_proxy_async();
    mbar_wait(bar_y, (uint32_t)s & 1, abort_flag, &g_tc_status, 71);
    float z[32];
    if (zy) {
      const uint8_t* yi = smem + OFF_Y;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int off = r * 128 + (((4 * h + c) ^ (r & 7)) << 4);
        const uint4 hi = *(const uint4*)(yi + off), lo = *(const uint4*)(yi + D * D * 2 + off);
        const uint32_t hw[4] = {hi.x, hi.y, hi.z, hi.w}, lw[4] = {lo.x, lo.y, lo.z, lo.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fh = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hw[e]));
          const float2 fl = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lw[e]));
          z[8 * c + 2 * e] = fh.x + fl.x;
          z[8 * c + 2 * e + 1] = fh.y + fl.y;
        }
      }
    }
    if (__syncthreads_or(*abort_flag != 0)) break;  // one decision for the CTA
    if (leader) {
      if (store_sfr && tprev >= 0) store_tile(g.bh * a.T + tprev);
      if (store_sst) store_tile(g.bh * a.nseg + s);
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t dxh = smem_desc_sw128(sb + OFF_XH + kk * 32, 16, 1024);
        const uint64_t dxl = smem_desc_sw128(sb + OFF_XL + kk * 32, 16, 1024);
        const uint64_t dyh = smem_desc_sw128(sb + OFF_Y + kk * 2048, D * 128, 1024);
        const uint64_t dyl = smem_desc_sw128(sb + OFF_Y + D * D * 2 + kk * 2048, D * 128, 1024);
        mma_bf16(tmem, dxh, dyh, idesc, kk > 0 ? 1u : 0u);
        mma_bf16(tmem, dxl, dyh, idesc, 1u);
        mma_bf16(tmem, dxh, dyl, idesc, 1u);
      }
      mma_commit(bar_mma);
    }
    mbar_wait(bar_mma, (uint32_t)s & 1, abort_flag, &g_tc_status, 72);
    tc_fence_after();
    if (leader && s + 1 < g.n) {
      fetch_y(chain_step_at(a, g, s + 1).Y);
      ++ny;
    }
    mbar_wait(bar_z, (uint32_t)s & 1, abort_flag, &g_tc_status, 73);
    if (!zy) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 f = *(const float4*)(smem + OFF_Z + h * 8192 + r * 128 + ((c ^ (r & 7)) << 4));
        z[4 * c] = f.x; z[4 * c + 1] = f.y; z[4 * c + 2] = f.z; z[4 * c + 3] = f.w;
      }
    }
    {
      uint32_t rr[32];
      tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + h * 32, rr);
      tmem_wait_ld();
      const float alpha = zy ? 1.0f : compose ? a.gamma[(size_t)g.bh * a.T + st.t] : st.alpha;
      if (active) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          x[c] = st.reset ? z[c] : alpha * (x[c] - __uint_as_float(rr[c])) + z[c];
      }
    }
    tc_fence_before();
    __syncthreads();  // every thread has read Z
    if (leader && s + 1 < g.n) {
      fetch_z(z_index(chain_step_at(a, g, s + 1)));
      ++nz;
    }
    if (compose) gprod *= a.gamma[(size_t)g.bh * a.T + st.t];
    if (store_sfr) {
      tprev = st.t;
      if (g.j0 + s == a.T - 1 && a.state_out && top)
        for (int c = 0; c < 32; ++c) a.state_out[(size_t)g.bh * DD + (size_t)r * D + h * 32 + c] = x[c];
    }
  }
  if ((store_sfr && tprev >= 0) || store_sst) {
    if (leader && nstore > 0) bulk_wait_read0();
    __syncthreads();
    if (!*abort_flag) {
      write_x();
      fence_proxy_async();
    }
    __syncthreads();
    if (leader && !*abort_flag) store_tile(store_sst ? g.bh * a.nseg + g.n : g.bh * a.T + tprev);
  }
  __syncthreads();
  if (!*abort_flag) {
    const size_t si = (size_t)g.bh * a.nseg + g.p;
    if (compose) {
      if (!top) {
        for (int c = 0; c < 32; ++c) a.Hc[si * DD + (size_t)r * D + h * 32 + c] = x[c];
      } else if (a.e_image) {
        uint8_t* img = (uint8_t*)a.E + si * c64::IMG;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int off = r * 128 + (((4 * h + c) ^ (r & 7)) << 4);
          split_chunk(x + 8 * c, (uint4*)(img + off), (uint4*)(img + D * D * 2 + off));
        }
      } else {
        for (int c = 0; c < 32; ++c) a.E[si * DD + (size_t)r * D + h * 32 + c] = x[c];
      }
      if (threadIdx.x == 0) a.g[si] = gprod;
    } else if (g.mode == CHAIN_PREFIX && !store_sst && top) {
      for (int c = 0; c < 32; ++c)
        a.Sst[((size_t)g.bh * a.nseg + g.n) * DD + (size_t)r * D + h * 32 + c] = x[c];
    }
  }
  if (leader) {
    if (nstore > 0) bulk_wait0();
    if (ny > 0) mbar_wait(bar_y, (uint32_t)(ny - 1) & 1, abort_flag, &g_tc_status, 74);
    if (nz > 0) mbar_wait(bar_z, (uint32_t)(nz - 1) & 1, abort_flag, &g_tc_status, 75);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// 3-D fp32 tensor of 64 x 64 matrices, box {32 columns, 64 rows}, 128-byte swizzle.
static cudaError_t make_map_f32_mats64(CUtensorMap* m, const void* base, uint64_t n) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {64, 64, n};
  cuuint64_t strides[2] = {64 * 4, 64 * 64 * 4};
  cuuint32_t box[3] = {32, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

static cudaError_t tc_chain64(const ChainArgs& a, int nchains, cudaStream_t st) {
  if (a.mode == CHAIN_SCAN && !a.sfr_hilo) return cudaErrorNotSupported;
  static DeviceOnce attr_once;
  const cudaError_t attr_status = once_per_device(attr_once, [&]() -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(k_chain64_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         h64::SMEM);
    return e;
  });
  if (attr_status != cudaSuccess) return attr_status;
  const long long frames = (long long)a.heads * a.T;
  CUtensorMap mz, ms;
  cudaError_t e = a.mode == CHAIN_PREFIX ? make_map_f32_mats64(&mz, a.Hc, (uint64_t)a.heads * a.nseg)
                                         : make_map_f32_mats64(&mz, a.U, (uint64_t)frames);
  if (e != cudaSuccess) return e;
  if (a.mode == CHAIN_PREFIX && a.sst_hilo)
    e = make_map_bf16_3d(&ms, a.Sst, 64, 64, 2 * (uint64_t)a.heads * a.nseg, 64, 64);
  else
    e = make_map_bf16_3d(&ms, a.mode == CHAIN_SCAN ? (const void*)a.Sfr : (const void*)a.U, 64, 64,
                         2 * frames, 64, 64);
  if (e != cudaSuccess) return e;
  // span composites run E and H stacked in one CTA per span
  const int grid = a.mode == CHAIN_COMPOSE ? nchains / 2 : nchains;
  k_chain64_tc<<<grid, h64::THREADS, h64::SMEM, st>>>(a, mz, ms);
  count_launch();
  return cudaGetLastError();
}

// ============================================================================
// Bidirectional readout (a6 for both directions, a1 fused), D = 128.
// Each raw Q tile is loaded once (and, with the prologue, transformed once)
// and multiplied with both directions' states:
//   O_fwd = Q S_fwd_hi^T + Q S_fwd_lo^T,   O_rev = Q S_rev_hi^T + Q S_rev_lo^T
// (four fp32 TMEM accumulators: two tiles in flight x two directions). Both
// outputs leave through two 16 KiB swizzled staging buffers and TMA stores.
// With the prologue, sixteen prologue warps transform every Q tile together
// and compute the RoPE angles (no room in shared memory for the table).
// ============================================================================
namespace rd2 {
constexpr int D = 128;
constexpr int TOK = 128;
constexpr int NQ = 2;
constexpr int BOX = TOK * 128;           // [128 rows][64 channels] bf16: 16 KiB
constexpr int QT = 2 * BOX;
constexpr int OFF_Q = 0;
constexpr int OFF_SF = OFF_Q + NQ * QT;  // forward state: hi (2 boxes), lo (2 boxes)
constexpr int OFF_SR = OFF_SF + 4 * BOX; // reverse state
constexpr int OFF_O = OFF_SR + 4 * BOX;  // two staging boxes
constexpr int OFF_W = OFF_O + 2 * BOX;   // prologue weights
constexpr int OFF_TH = OFF_W + D * 4;    // prologue pair frequencies [D/4]
constexpr int OFF_BAR = OFF_TH + (D / 4) * 4;
constexpr int NBAR = 3 * NQ + 2 + 4 + 1;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM = OFF_MISC + 16 + 1024;
static_assert(SMEM <= 232448, "bidirectional readout shared memory");
constexpr int threads(bool pro) { return pro ? 704 : 192; }  // + 16 prologue warps
constexpr uint32_t TMEM_COLS = 512;
}  // namespace rd2

template <bool PRO, bool UC = false>
__global__ void __launch_bounds__(rd2::threads(PRO), 1)
    k_readout2_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmSF,
                  const __grid_constant__ CUtensorMap tmSR, const __grid_constant__ CUtensorMap tmOF,
                  const __grid_constant__ CUtensorMap tmOR, int N, int S, ProArgs pro,
                  int parts) {
  using namespace rd2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_qf = sb + OFF_BAR;
  const uint32_t bar_qr = bar_qf + 8 * NQ;
  const uint32_t bar_qe = bar_qr + 8 * NQ;
  const uint32_t bar_sf = bar_qe + 8 * NQ;
  const uint32_t bar_se = bar_sf + 8;
  const uint32_t bar_accf = bar_se + 8;
  const uint32_t bar_acce = bar_accf + 16;
  const uint32_t bar_fin = bar_acce + 16;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  if (threadIdx.x == 0) {
    for (int s = 0; s < NQ; ++s) {
      mbar_init(bar_qf + 8 * s, 1);
      mbar_init(bar_qr + 8 * s, 16);  // every prologue warp
      mbar_init(bar_qe + 8 * s, 1);
    }
    mbar_init(bar_sf, 1);
    mbar_init(bar_se, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf + 8 * b, 1);
      mbar_init(bar_acce + 8 * b, 4);  // every epilogue warp
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (PRO) pro_w_copy((float2*)(smem + OFF_W), pro.w);
  if (PRO && threadIdx.x < D / 4)  // pair frequencies, as the (cos, sin) table has them
    ((float*)(smem + OFF_TH))[threadIdx.x] =
        rope_theta(pro.base, threadIdx.x, pro.ucpe ? D / 2 : D);  // entries 0-15 with the camera
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int ntile = (S + TOK - 1) / TOK;
  // Work units: each frame-head's tiles in kParts contiguous parts (outputs are
  // per token, so parts need no reduction); finer units even out the rounds.
  const int kParts = parts;
  const int NU = N * kParts;
  const int my_count = (int)blockIdx.x < NU ? (NU - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp == 0) {
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_count && ok; ++i) {
        const int unit = blockIdx.x + i * gridDim.x;
        const int n = unit / kParts, part = unit % kParts;
        const int tl0 = part * ntile / kParts, tl1 = (part + 1) * ntile / kParts;
        (void)n;
                ok = mbar_wait(bar_se, ((uint32_t)i & 1) ^ 1, abort_flag, &g_tc_status, 81);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_sf, 8 * BOX);
        // [S_f ; S_r] as one K-major N = 256 operand: per hi / lo half, per
        // 64-channel block x, the 128 rows of S_f then the 128 rows of S_r
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const uint32_t dst = sb + OFF_SF + hl * 4 * BOX + x * 2 * BOX;
            tma_load_3d(dst, &tmSF, bar_sf, 64 * x, 0, 2 * n + hl);
            tma_load_3d(dst + BOX, &tmSR, bar_sf, 64 * x, 0, 2 * n + hl);
          }
        for (int tl = tl0; tl < tl1; ++tl, ++g) {
          const int s = g % NQ;
          const uint32_t u = (uint32_t)(g / NQ);
          ok = mbar_wait(bar_qe + 8 * s, (u & 1) ^ 1, abort_flag, &g_tc_status, 82);
          if (!ok) break;
          const uint32_t qd = sb + OFF_Q + s * QT;
          mbar_arrive_expect_tx(bar_qf + 8 * s, QT);
          tma_load_3d(qd, &tmQ, bar_qf + 8 * s, 0, tl * TOK, n);
          tma_load_3d(qd + BOX, &tmQ, bar_qf + 8 * s, 64, tl * TOK, n);
        }
      }
      for (int gg = (g > NQ ? g - NQ : 0); gg < g; ++gg)
        mbar_wait(bar_qf + 8 * (gg % NQ), (uint32_t)(gg / NQ) & 1, abort_flag, &g_tc_status, 83);
      if (my_count > 0) mbar_wait(bar_sf, (uint32_t)(my_count - 1) & 1, abort_flag, &g_tc_status, 84);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256, false, false);
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_count && ok; ++i) {
        const int unit = blockIdx.x + i * gridDim.x;
        const int n = unit / kParts, part = unit % kParts;
        const int tl0 = part * ntile / kParts, tl1 = (part + 1) * ntile / kParts;
        (void)n;
        ok = mbar_wait(bar_sf, (uint32_t)i & 1, abort_flag, &g_tc_status, 85);
        if (!ok) break;
        tc_fence_after();
        for (int tl = tl0; tl < tl1; ++tl, ++g) {
          const int s = g % NQ;
          const uint32_t u = (uint32_t)(g / NQ);
          const int b = g & 1;
          const uint32_t ub = (uint32_t)(g >> 1);
          ok = mbar_wait(bar_acce + 8 * b, (ub & 1) ^ 1, abort_flag, &g_tc_status, 86);
          if (!ok) break;
          ok = mbar_wait((PRO ? bar_qr : bar_qf) + 8 * s, u & 1, abort_flag, &g_tc_status, 87);
          if (!ok) break;
          tc_fence_after();
          const uint32_t qa = sb + OFF_Q + s * QT;
          // [O_f | O_r] = Q [S_f ; S_r]^T: one N = 256 MMA per 16 channels and half
          const uint32_t d = tmem + b * 256;
          const uint32_t sh = sb + OFF_SF, sl = sh + 4 * BOX;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * BOX + (kk & 3) * 32;
            const uint32_t soff = (kk >> 2) * 2 * BOX + (kk & 3) * 32;
            const uint64_t dq = smem_desc_sw128(qa + off, 16, 1024);
            mma_bf16(d, dq, smem_desc_sw128(sh + soff, 16, 1024), idesc, kk > 0 ? 1u : 0u);
            mma_bf16(d, dq, smem_desc_sw128(sl + soff, 16, 1024), idesc, 1u);
          }
          mma_commit(bar_qe + 8 * s);
          mma_commit(bar_accf + 8 * b);
        }
        if (!ok) break;
        mma_commit(bar_se);
      }
      mma_commit(bar_fin);
      mbar_wait(bar_fin, 0, abort_flag, &g_tc_status, 88);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ---- epilogue: four 64-column rounds per tile (fwd lo/hi half, rev ...) ----
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int et = threadIdx.x - 64;
    int g = 0, nstores = 0;
    bool ok = true;
    for (int i = 0; i < my_count && ok; ++i) {
      const int unit = blockIdx.x + i * gridDim.x;
      const int n = unit / kParts, part = unit % kParts;
      const int tl0 = part * ntile / kParts, tl1 = (part + 1) * ntile / kParts;
      (void)n;
            for (int tl = tl0; tl < tl1; ++tl, ++g) {
        const int b = g & 1;
        const uint32_t ub = (uint32_t)(g >> 1);
        mbar_wait(bar_accf + 8 * b, ub & 1, abort_flag, &g_tc_status, 89);
        tc_fence_after();
#pragma unroll
        for (int rnd = 0; rnd < 4; ++rnd) {
          const int dir = rnd >> 1, half = rnd & 1, buf = nstores & 1;
          // the store that last used this staging buffer has read it
          if (et == 0 && nstores >= 2) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
          if (named_bar_or(1, 128, *abort_flag != 0)) {
            ok = false;
            break;
          }
          uint8_t* ost = smem + OFF_O + buf * BOX;
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + b * 256 + dir * 128 + half * 64 + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 4; ++j)
              *(uint4*)(ost + row * 128 + ((((c0 >> 3) + j) ^ (row & 7)) << 4)) = make_uint4(
                  pack_bf16x2(__uint_as_float(r[8 * j]), __uint_as_float(r[8 * j + 1])),
                  pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3])),
                  pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5])),
                  pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7])));
          }
          fence_proxy_async();
          named_bar_sync(1, 128);
          if (et == 0) {
            tma_store_3d(dir ? &tmOR : &tmOF, sb + OFF_O + buf * BOX, 64 * half, tl * TOK, n);
            bulk_commit();
          }
          ++nstores;
        }
        if (!ok) break;
        tc_fence_before();
        warp_arrive(bar_acce + 8 * b);
      }
    }
    if (et == 0) bulk_wait0();
  } else if (PRO) {
    // all sixteen prologue warps on every Q tile: four threads per token
    // (32 channels each), one token each
    const int t = threadIdx.x - 192;
    const int pr = pro_lane_row(t), pq = pro_lane_quarter(t);
    int g = 0;
    bool ok = true;
    for (int i = 0; i < my_count && ok; ++i) {
      const int unit = blockIdx.x + i * gridDim.x;
      const int n = unit / kParts, part = unit % kParts;
      const int tl0 = part * ntile / kParts, tl1 = (part + 1) * ntile / kParts;
      (void)n;
      for (int tl = tl0; tl < tl1; ++tl, ++g) {
        const int s = g % NQ;
        const uint32_t u = (uint32_t)(g / NQ);
        ok = mbar_wait(bar_qf + 8 * s, u & 1, abort_flag, &g_tc_status, 90);
        if (!ok) break;
        const int rr[1] = {pr}, tk[1] = {tl * TOK + pr};
        const float bv[1] = {1.f};
        pro_rows<1, true, false, UC>(smem + OFF_Q + s * QT, BOX, rr, pq, tk, S, pro,
                                 (const float2*)(smem + OFF_W), nullptr, (const float*)(smem + OFF_TH),
                                 nullptr, bv, n);
        fence_proxy_async();
        warp_arrive(bar_qr + 8 * s);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <bool PRO, bool UC = false>
static cudaError_t launch_readout2(const CUtensorMap* m, long long N, int S, const ProArgs& pa,
                                   cudaStream_t st) {
  static DeviceOnce attr_once;
  const cudaError_t attr_status = once_per_device(attr_once, [&]() -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(k_readout2_tc<PRO, UC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         rd2::SMEM);
    return e;
  });
  if (attr_status != cudaSuccess) return attr_status;
  const int parts = readout_parts(N, (S + rd2::TOK - 1) / rd2::TOK);
  const long long units = N * parts;
  const int grid = (int)(units < num_sms() ? units : num_sms());
  k_readout2_tc<PRO, UC><<<grid, rd2::threads(PRO), rd2::SMEM, st>>>(m[0], m[1], m[2], m[3], m[4],
                                                                      (int)N, S, pa, parts);
  count_launch();
  return cudaGetLastError();
}

bool tc_readout2_supported(int D) { return D == 128; }

cudaError_t tc_readout2(const void* q, const void* sfr_f, const void* sfr_r, void* out_f,
                        void* out_r, long long N, int S, int D, const ProArgs* pro,
                        cudaStream_t st) {
  if (D != 128) return cudaErrorNotSupported;
  CUtensorMap m[5];
  cudaError_t e = make_map_bf16_3d(&m[0], q, D, S, N, 64, rd2::TOK);
  if (e == cudaSuccess) e = make_map_bf16_3d(&m[1], sfr_f, D, D, 2 * N, 64, 128);
  if (e == cudaSuccess) e = make_map_bf16_3d(&m[2], sfr_r, D, D, 2 * N, 64, 128);
  if (e == cudaSuccess) e = make_map_bf16_3d(&m[3], out_f, D, S, N, 64, rd2::TOK);
  if (e == cudaSuccess) e = make_map_bf16_3d(&m[4], out_r, D, S, N, 64, rd2::TOK);
  if (e != cudaSuccess) return e;
  ProArgs pa = {};
  if (pro) {
    pa = *pro;
    if (pa.ucpe) return launch_readout2<true, true>(m, N, S, pa, st);
    return launch_readout2<true>(m, N, S, pa, st);
  }
  return launch_readout2<false>(m, N, S, pa, st);
}

// ============================================================================
// D = 256 tensor-core contraction and readout, each on CTA pairs (clusters of
// two CTAs sharing one tcgen05 MMA of M = 256): every byte of K, V and Q is
// loaded by one CTA only and multiplied once.
// ============================================================================
__device__ __forceinline__ int img256_off(int k, int n8);

// D = 256 contraction on a CTA pair (a cluster of two CTAs, one tcgen05
// MMA of M = 256 over both). Per frame-head and 64-token stage CTA r of the
// pair loads only channels 128r .. 128r + 127 of K and of V (TMA, 128-byte
// swizzle, evict-first) and scales its K half by beta; the even CTA then
// issues, per 16 tokens,
//     A += K^T (beta K),  U += V^T (beta K)        (M = 256, N = 256, K = 16)
// with the A operands (K, V) split by rows and the B operand (beta K) split
// by columns over the two CTAs' shared memory, so each byte of K and V is
// read from memory once and multiplied once. CTA r's TMEM receives rows
// 128r .. of A (columns 0-255) and of U (256-511); its eight epilogue warps
// (four on A, four on U) write rows 128r .. of A_t as the bf16 (hi, lo)
// operand image of the D = 256 chains and of U_t transposed (or both in fp32
// when no image is asked for). Barriers: stage
// and beta*K slot releases are multicast MMA commits to both CTAs. The even
// CTA's scalers arrive on its slot barrier directly; the odd CTA's arrive on
// a local barrier, and a relay warp per slot forwards each completed use of
// it with one cluster-scope arrival, so the scaler warps never wait on a
// cluster-wide release and the releases of successive stages overlap. The epilogue warps of both CTAs arrive on the even
// CTA's accumulator barrier. The MMA thread thus starts a stage once both
// halves of its beta*K are written and a unit once both CTAs have drained
// their accumulators.
namespace cp256 {
constexpr int D = 256;
constexpr int TOK = 64;                 // tokens per stage
constexpr int NST = 5;                  // stages
constexpr int NBK = 4;                  // beta * K slots (each stage's slot waits for the
                                        // pair's MMAs NBK stages back, across both CTAs)
constexpr int BOX = TOK * 128;          // [64 tokens][64 channels]: 8 KiB
constexpr int HT = 2 * BOX;             // this CTA's 128 channels of a stage: 16 KiB
constexpr int OFF_K = 0;
constexpr int OFF_V = OFF_K + NST * HT;
constexpr int OFF_BK = OFF_V + NST * HT;
constexpr int OFF_BETA = OFF_BK + NBK * HT;
constexpr int OFF_BAR = OFF_BETA + NST * TOK * 4;
constexpr int NBAR = 2 * NST + 3 * NBK + 3;  // full, empty; bk_full, bk_empty, bk_local; acc f/e, fin
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM = OFF_MISC + 16 + 1024;
static_assert(SMEM <= 232448, "D = 256 pair contraction shared memory");
constexpr int NSC = 128;                // scaler threads
constexpr int NEPI = 8;                 // epilogue warps
constexpr int NRELAY = NBK;             // relay warps of the odd CTA, one per slot
constexpr int THREADS = 64 + NSC + 32 * NEPI + 32 * NRELAY;
constexpr uint32_t TMEM_COLS = 512;
static_assert((HT / 16) % NSC == 0, "scaler chunks");
}  // namespace cp256

__global__ void __launch_bounds__(cp256::THREADS, 1)
    k_contract256_pair_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const float* __restrict__ beta, float* __restrict__ A, float* __restrict__ U,
                          int N, int S, float cA, float cU, int a_image) {
  using namespace cp256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the pair's MMAs
  const uint32_t bar_full = sb + OFF_BAR;
  const uint32_t bar_empty = bar_full + 8 * NST;
  const uint32_t bar_bkf = bar_empty + 8 * NST;
  const uint32_t bar_bke = bar_bkf + 8 * NBK;
  const uint32_t bar_bkl = bar_bke + 8 * NBK;
  const uint32_t bar_accf = bar_bkl + 8 * NBK;
  const uint32_t bar_acce = bar_accf + 8;
  const uint32_t bar_fin = bar_acce + 8;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full + 8 * s, 33);  // expect_tx + 32 lanes' beta copies
      mbar_init(bar_empty + 8 * s, 1);  // the pair's MMA commit
    }
    for (int s = 0; s < NBK; ++s) {
      mbar_init(bar_bkf + 8 * s, NSC / 32 + 1);  // this CTA's scaler warps + the odd CTA's relay
      mbar_init(bar_bke + 8 * s, 1);
      mbar_init(bar_bkl + 8 * s, NSC / 32);      // the odd CTA's scaler warps
    }
    mbar_init(bar_accf, 1);
    mbar_init(bar_acce, 2 * NEPI);  // the epilogue warps of both CTAs
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before either arrives on the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int nst_frame = (S + TOK - 1) / TOK;
  const int pair = (int)blockIdx.x >> 1, npair = (int)gridDim.x >> 1;
  const int my_count = pair < N ? (N - 1 - pair) / npair + 1 : 0;

  if (warp == 0) {
    const uint64_t pol = l2_policy_evict_first();  // K and V are read once
    int g = 0;
    bool ok = true;
    for (int i = 0; i < my_count && ok; ++i) {
      const int n = pair + i * npair;
      for (int st = 0; st < nst_frame; ++st, ++g) {
        const int s = g % NST;
        const uint32_t u = (uint32_t)(g / NST);
        if (lane == 0) ok = mbar_wait(bar_empty + 8 * s, (u & 1) ^ 1, abort_flag, &g_tc_status, 121);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(bar_full + 8 * s, 2 * HT);
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const int ch = 128 * (int)rank + 64 * x;
            tma_load_3d_hint(sb + OFF_K + s * HT + x * BOX, &tmK, bar_full + 8 * s, ch, st * TOK, n, pol);
            tma_load_3d_hint(sb + OFF_V + s * HT + x * BOX, &tmV, bar_full + 8 * s, ch, st * TOK, n, pol);
          }
        }
        const uint32_t bsa = sb + OFF_BETA + s * TOK * 4;
#pragma unroll
        for (int r = lane; r < TOK; r += 32) {
          const int tok = st * TOK + r;
          const bool in = tok < S;
          cp_async_4(bsa + r * 4, beta + (size_t)n * S + (in ? tok : 0), in ? 4u : 0u);
        }
        cp_async_arrive_noinc(bar_full + 8 * s);
      }
    }
    if (lane == 0)
      for (int gg = (g > NST ? g - NST : 0); gg < g; ++gg)
        mbar_wait(bar_full + 8 * (gg % NST), (uint32_t)(gg / NST) & 1, abort_flag, &g_tc_status, 122);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, 256, true, true);
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_count && ok; ++i) {
        ok = mbar_wait_cluster(bar_acce, ((uint32_t)i & 1) ^ 1, abort_flag, &g_tc_status, 123);
        if (!ok) break;
        tc_fence_after();
        for (int st = 0; st < nst_frame; ++st, ++g) {
          const int s = g % NST, kb = g % NBK;
          ok = mbar_wait_cluster(bar_bkf + 8 * kb, (uint32_t)(g / NBK) & 1, abort_flag, &g_tc_status, 124);
          if (!ok) break;
          tc_fence_after();
          const uint32_t ka = sb + OFF_K + s * HT, va = sb + OFF_V + s * HT, ba = sb + OFF_BK + kb * HT;
#pragma unroll
          for (int kk = 0; kk < TOK / 16; ++kk) {
            const uint64_t db = smem_desc_sw128(ba + kk * 2048, BOX, 1024);
            const uint32_t acc = (st > 0 || kk > 0) ? 1u : 0u;
            mma_bf16_pair(tmem, smem_desc_sw128(ka + kk * 2048, BOX, 1024), db, idesc, acc);
            mma_bf16_pair(tmem + 256, smem_desc_sw128(va + kk * 2048, BOX, 1024), db, idesc, acc);
          }
          mma_commit_pair(bar_empty + 8 * s, 3);
          mma_commit_pair(bar_bke + 8 * kb, 3);
        }
        if (!ok) break;
        mma_commit_pair(bar_accf, 3);
      }
      mma_commit_pair(bar_fin, 3);
    }
    __syncwarp();
  } else if (warp >= 2 + NSC / 32 + NEPI) {
    // relay warp kb of the odd CTA: forwards each use of beta * K slot kb that
    // this CTA's scalers completed to the even CTA's slot barrier
    const int kb = warp - (2 + NSC / 32 + NEPI);
    if (rank != 0 && lane == 0) {
      const uint32_t bkf_lead = mapa_shared(bar_bkf + 8 * kb, 0);
      const int total = my_count * nst_frame;  // stages kb, kb + NBK, ... of this CTA
      for (int g = kb, u = 0; g < total; g += NBK, ++u) {
        if (!mbar_wait(bar_bkl + 8 * kb, (uint32_t)u & 1, abort_flag, &g_tc_status, 129)) break;
        mbar_arrive_cluster(bkf_lead);
      }
    }
    __syncwarp();
  } else if (warp < 2 + NSC / 32) {
    const int t = threadIdx.x - 64;
    const uint32_t bar_done = rank == 0 ? bar_bkf : bar_bkl;  // see the relay warps
    int g = 0;
    bool ok = true;
    for (int i = 0; i < my_count && ok; ++i) {
      for (int st = 0; st < nst_frame; ++st, ++g) {
        const int s = g % NST, kb = g % NBK;
        const uint32_t u = (uint32_t)(g / NST);
        ok = mbar_wait(bar_full + 8 * s, u & 1, abort_flag, &g_tc_status, 125);
        // the slot's previous beta * K has been consumed by the pair's MMAs
        if (ok) ok = mbar_wait(bar_bke + 8 * kb, ((uint32_t)(g / NBK) & 1) ^ 1, abort_flag, &g_tc_status, 126);
        if (!ok) break;
        const uint8_t* kt = smem + OFF_K + s * HT;
        uint8_t* bt = smem + OFF_BK + kb * HT;
        const float* bs = (const float*)(smem + OFF_BETA) + s * TOK;
#pragma unroll
        for (int m = 0; m < (HT / 16) / NSC; ++m) {
          const int c = t + NSC * m;
          const float bv = bs[(c >> 3) & (TOK - 1)];
          const uint4 x = *(const uint4*)(kt + c * 16);
          uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w[e]));
            w[e] = pack_bf16x2(f.x * bv, f.y * bv);
          }
          *(uint4*)(bt + c * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async();
        warp_arrive(bar_done + 8 * kb);
      }
    }
  } else {
    const int q = warp & 3;
    const int mat = (warp - 2 - NSC / 32) >> 2;  // 0: A, 1: U
    const int row = q * 32 + lane;
    const int k = 128 * (int)rank + row;
    const uint32_t acce_lead = mapa_shared(bar_acce, 0);
    const float sc = mat ? cU : cA;
    for (int i = 0; i < my_count; ++i) {
      const int n = pair + i * npair;
      if (!mbar_wait(bar_accf, (uint32_t)i & 1, abort_flag, &g_tc_status, 127)) break;
      tc_fence_after();
      float* dst = (mat ? U : A) + ((size_t)n * D + k) * D;
      uint8_t* img = (uint8_t*)A + (size_t)n * D * D * 4;
      for (int c0 = 0; c0 < 256; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + mat * 256 + c0, r);
        tmem_wait_ld();
        if (mat == 0 && a_image) {
          // row k of A_t into the operand image (hi, lo) of the D = 256 chains
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(r[8 * j + e]) * sc;
            uint4 hi, lo;
            split_chunk(v, &hi, &lo);
            const int off = img256_off(k, (c0 >> 3) + j);
            *(uint4*)(img + off) = hi;
            *(uint4*)(img + off + 8192) = lo;
          }
        } else if (mat == 1 && a_image) {
          // U_t transposed for the D = 256 chains
          float* ut = U + (size_t)n * D * D + k;
#pragma unroll
          for (int j = 0; j < 32; ++j) ut[(size_t)(c0 + j) * D] = __uint_as_float(r[j]) * sc;
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *(float4*)(dst + c0 + 4 * j) =
                make_float4(__uint_as_float(r[4 * j]) * sc, __uint_as_float(r[4 * j + 1]) * sc,
                            __uint_as_float(r[4 * j + 2]) * sc, __uint_as_float(r[4 * j + 3]) * sc);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acce_lead);
    }
  }
  // Teardown: every MMA of the pair has completed (bar_fin, multicast), and
  // neither CTA leaves while the other may still arrive on its barriers.
  tc_fence_before();
  __syncthreads();
  if (warp == 1 && lane == 0) {
    volatile int keep_waiting = 0;
    mbar_wait(bar_fin, 0, &keep_waiting, &g_tc_status, 128);
  }
  __syncwarp();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// D = 256 readout on a CTA pair: tiles of 256 tokens, CTA r of the pair
// loading tokens 128r .. 128r + 127 of each (all 256 channels, as four
// 64-channel stages of a four-stage ring) and holding rows 128r .. of S_t
// (hi, lo: 128 KiB). The even CTA issues O = Q S_hi^T + Q S_lo^T as M = 256
// (tokens, split over the pair), N = 256 (columns of O, split over the pair's
// S halves) MMAs, so each Q tile is read once; CTA r's TMEM receives its 128
// tokens x 256 columns (double-buffered: 2 x 256 columns), read by its eight
// epilogue warps (two per TMEM lane quarter, 128 columns each) in one batch
// of TMEM loads, released to the MMA, then written back in four passes of
// 64 columns through two 16 KiB staging boxes taken in turn, each pass one
// TMA store. Both CTAs' Q and S loads complete their bytes on
// the even CTA's barriers (the odd CTA's through the pair form of the TMA
// load), which expect the bytes of both; stage and S releases are multicast
// MMA commits; each CTA's epilogue signals the even CTA once per tile.
namespace rp256 {
constexpr int D = 256;
constexpr int TOK = 128;                 // tokens per CTA and tile (256 per pair)
constexpr int NQ = 4;                    // Q stages of 64 channels (four per tile)
constexpr int BOX = TOK * 128;           // [128 rows][64 channels]: 16 KiB
static_assert(4 * BOX == TOK * D * 2, "four stages hold a tile's D bf16 channels");
constexpr int OFF_Q = 0;
constexpr int OFF_S = OFF_Q + NQ * BOX;  // S rows half: hi 4 boxes, lo 4 boxes (128 KiB)
constexpr int OFF_O = OFF_S + 8 * BOX;   // output staging: two boxes, used in turn
constexpr int OFF_BAR = OFF_O + 2 * BOX;
constexpr int NBAR = 2 * NQ + 2 + 4 + 1;  // qf, qe; sf, se; accf x2, acce x2; fin
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM = OFF_MISC + 16 + 1024;
static_assert(SMEM <= 232448, "D = 256 pair readout shared memory");
constexpr int NEPI = 8;                  // epilogue warps
constexpr int THREADS = 64 + 32 * NEPI;
constexpr uint32_t TMEM_COLS = 512;
}  // namespace rp256

__global__ void __launch_bounds__(rp256::THREADS, 1)
    k_readout256_pair_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmS,
                         const __grid_constant__ CUtensorMap tmO, int N, int S) {
  using namespace rp256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the pair's MMAs
  const uint32_t bar_qf = sb + OFF_BAR;
  const uint32_t bar_qe = bar_qf + 8 * NQ;
  const uint32_t bar_sf = bar_qe + 8 * NQ;
  const uint32_t bar_se = bar_sf + 8;
  const uint32_t bar_accf = bar_se + 8;
  const uint32_t bar_acce = bar_accf + 16;
  const uint32_t bar_fin = bar_acce + 16;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  if (threadIdx.x == 0) {
    for (int s = 0; s < NQ; ++s) {
      mbar_init(bar_qf + 8 * s, 1);  // the even CTA's expect; the bytes of both CTAs
      mbar_init(bar_qe + 8 * s, 1);
    }
    mbar_init(bar_sf, 1);
    mbar_init(bar_se, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf + 8 * b, 1);
      mbar_init(bar_acce + 8 * b, 2);  // one arrival per CTA
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before either arrives on the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int ntile = (S + 2 * TOK - 1) / (2 * TOK);
  const int pair = (int)blockIdx.x >> 1, npair = (int)gridDim.x >> 1;
  const int my_count = pair < N ? (N - 1 - pair) / npair + 1 : 0;

  if (warp == 0) {
    if (lane == 0) {
      // loads land in this CTA's shared memory; their bytes complete on the
      // even CTA's barriers
      const uint32_t qf_lead = mapa_shared(bar_qf, 0), sf_lead = mapa_shared(bar_sf, 0);
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_count && ok; ++i) {
        const int n = pair + i * npair;
        ok = mbar_wait(bar_se, ((uint32_t)i & 1) ^ 1, abort_flag, &g_tc_status, 131);
        if (!ok) break;
        if (rank == 0) mbar_arrive_expect_tx(bar_sf, 2 * 8 * BOX);
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int x = 0; x < 4; ++x)
            tma_load_3d_pair(sb + OFF_S + (4 * hl + x) * BOX, &tmS, sf_lead, 64 * x, 128 * (int)rank,
                             2 * n + hl);
        for (int tl = 0; tl < ntile && ok; ++tl)
          for (int qq = 0; qq < 4; ++qq, ++g) {
            const int s = g % NQ;
            const uint32_t u = (uint32_t)(g / NQ);
            ok = mbar_wait(bar_qe + 8 * s, (u & 1) ^ 1, abort_flag, &g_tc_status, 132);
            if (!ok) break;
            const int tok0 = 2 * TOK * tl + TOK * (int)rank;  // may lie past S: zero fill
            if (rank == 0) mbar_arrive_expect_tx(bar_qf + 8 * s, 2 * BOX);
            tma_load_3d_pair(sb + OFF_Q + s * BOX, &tmQ, qf_lead + 8 * s, 64 * qq, tok0, n);
          }
      }
      // the even CTA's barriers count both CTAs' bytes: its drain covers the pair
      if (rank == 0) {
        for (int gg = (g > NQ ? g - NQ : 0); gg < g; ++gg)
          mbar_wait(bar_qf + 8 * (gg % NQ), (uint32_t)(gg / NQ) & 1, abort_flag, &g_tc_status, 133);
        if (my_count > 0) mbar_wait(bar_sf, (uint32_t)(my_count - 1) & 1, abort_flag, &g_tc_status, 134);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, 256, false, false);
      int g = 0, gt = 0;
      bool ok = true;
      for (int i = 0; i < my_count && ok; ++i) {
        ok = mbar_wait(bar_sf, (uint32_t)i & 1, abort_flag, &g_tc_status, 135);
        if (!ok) break;
        tc_fence_after();
        for (int tl = 0; tl < ntile && ok; ++tl, ++gt) {
          const int b = gt & 1;
          const uint32_t ub = (uint32_t)(gt >> 1);
          ok = mbar_wait_cluster(bar_acce + 8 * b, (ub & 1) ^ 1, abort_flag, &g_tc_status, 137);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tmem + b * 256;
          for (int qq = 0; qq < 4 && ok; ++qq, ++g) {
            const int s = g % NQ;
            ok = mbar_wait(bar_qf + 8 * s, (uint32_t)(g / NQ) & 1, abort_flag, &g_tc_status, 138);
            if (!ok) break;
            tc_fence_after();
            const uint32_t qa = sb + OFF_Q + s * BOX;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t soff = qq * BOX + kk * 32;
              const uint64_t dq = smem_desc_sw128(qa + kk * 32, 16, 1024);
              mma_bf16_pair(d, dq, smem_desc_sw128(sb + OFF_S + soff, 16, 1024), idesc,
                            (qq > 0 || kk > 0) ? 1u : 0u);
              mma_bf16_pair(d, dq, smem_desc_sw128(sb + OFF_S + 4 * BOX + soff, 16, 1024), idesc, 1u);
            }
            mma_commit_pair(bar_qe + 8 * s, 3);
          }
          if (!ok) break;
          mma_commit_pair(bar_accf + 8 * b, 3);
        }
        if (!ok) break;
        mma_commit_pair(bar_se, 3);
      }
      mma_commit_pair(bar_fin, 3);
    }
    __syncwarp();
  } else {
    const int q = warp & 3;                // TMEM lane quarter
    const int h = (warp - 2) >> 2;         // 32-column half of a pass
    const int row = q * 32 + lane;
    const int et = threadIdx.x - 64;
    constexpr int NET = 32 * NEPI;
    const uint32_t acce_lead = mapa_shared(bar_acce, 0);
    int gt = 0, npass = 0;
    bool ok = true;
    for (int i = 0; i < my_count && ok; ++i) {
      const int n = pair + i * npair;
      for (int tl = 0; tl < ntile; ++tl, ++gt) {
        const int b = gt & 1;
        const uint32_t ub = (uint32_t)(gt >> 1);
        const int tok0 = 2 * TOK * tl + TOK * (int)rank;
        mbar_wait(bar_accf + 8 * b, ub & 1, abort_flag, &g_tc_status, 142);
        tc_fence_after();
        // the thread's 128 columns (four passes of 32) in one batch of TMEM
        // loads; the buffer is released to the MMA before any store
        uint32_t r[4][32];
#pragma unroll
        for (int p = 0; p < 4; ++p)
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + b * 256 + p * 64 + 32 * h, r[p]);
        tmem_wait_ld();
        tc_fence_before();
#pragma unroll
        for (int p = 0; p < 4; ++p, ++npass) {
          // the store that last used this staging box (two passes back) has read it
          if (et == 0 && npass >= 2) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
          if (named_bar_or(1, NET, *abort_flag != 0)) {
            ok = false;
            break;
          }
          // every epilogue thread of this CTA has read the accumulator
          if (p == 0 && et == 32) mbar_arrive_cluster(acce_lead + 8 * b);
          uint8_t* ost = smem + OFF_O + (npass & 1) * BOX;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *(uint4*)(ost + row * 128 + (((4 * h + j) ^ (row & 7)) << 4)) = make_uint4(
                pack_bf16x2(__uint_as_float(r[p][8 * j]), __uint_as_float(r[p][8 * j + 1])),
                pack_bf16x2(__uint_as_float(r[p][8 * j + 2]), __uint_as_float(r[p][8 * j + 3])),
                pack_bf16x2(__uint_as_float(r[p][8 * j + 4]), __uint_as_float(r[p][8 * j + 5])),
                pack_bf16x2(__uint_as_float(r[p][8 * j + 6]), __uint_as_float(r[p][8 * j + 7])));
          fence_proxy_async();
          named_bar_sync(1, NET);
          if (et == 0) {
            if (tok0 < S) tma_store_3d(&tmO, smem_u32(ost), 64 * p, tok0, n);
            bulk_commit();  // one group per pass, empty past S, so the waits above count passes
          }
        }
        if (!ok) break;
      }
    }
    if (et == 0) bulk_wait0();
  }
  // Teardown: every MMA of the pair has completed (bar_fin, multicast), and
  // neither CTA leaves while the other may still arrive on its barriers.
  tc_fence_before();
  __syncthreads();
  if (warp == 1 && lane == 0) {
    volatile int keep_waiting = 0;
    mbar_wait(bar_fin, 0, &keep_waiting, &g_tc_status, 143);
  }
  __syncwarp();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// Clusters of two CTAs of `kernel` (with `smem` bytes of dynamic shared
// memory each) that can be resident at once; 0 if none.
template <class K>
static int max_active_pairs(K kernel, int threads, int smem) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * num_sms());
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

template <class K, class... Args>
static cudaError_t launch_pairs(K kernel, int npair, int threads, int smem, cudaStream_t st,
                                Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * npair);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

static cudaError_t tc_contract256(const void* k, const void* v, const float* beta, float* A,
                                  float* U, long long N, int S, float cA, float cU, int a_image,
                                  cudaStream_t st) {
  static DeviceOnce pair_once;
  static int pairs_per_dev[64];
  int dev = 0;
  cudaGetDevice(&dev);
  const cudaError_t pe = once_per_device(pair_once, [&]() -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(k_contract256_pair_tc,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, cp256::SMEM);
    if (e != cudaSuccess) return e;
    pairs_per_dev[dev & 63] = max_active_pairs(k_contract256_pair_tc, cp256::THREADS, cp256::SMEM);
    return cudaSuccess;
  });
  if (pe != cudaSuccess) return pe;
  const int maxp = pairs_per_dev[dev & 63];
  if (maxp <= 0) return cudaErrorNotSupported;  // no cluster of two can be resident
  CUtensorMap mk, mv;
  cudaError_t e = make_map_bf16_3d(&mk, k, 256, S, N, 64, cp256::TOK);
  if (e == cudaSuccess) e = make_map_bf16_3d(&mv, v, 256, S, N, 64, cp256::TOK);
  if (e != cudaSuccess) return e;
  const int npair = (int)(N < maxp ? N : maxp);
  e = launch_pairs(k_contract256_pair_tc, npair, cp256::THREADS, cp256::SMEM, st, mk, mv, beta, A, U,
                   (int)N, S, cA, cU, a_image);
  count_launch();
  return e;
}

static cudaError_t tc_readout256(const void* q, const void* Sfr_hilo, void* out, long long N, int S,
                                 cudaStream_t st) {
  static DeviceOnce pair_once;
  static int pairs_per_dev[64];
  int dev = 0;
  cudaGetDevice(&dev);
  const cudaError_t pe = once_per_device(pair_once, [&]() -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(k_readout256_pair_tc,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, rp256::SMEM);
    if (e != cudaSuccess) return e;
    pairs_per_dev[dev & 63] = max_active_pairs(k_readout256_pair_tc, rp256::THREADS, rp256::SMEM);
    return cudaSuccess;
  });
  if (pe != cudaSuccess) return pe;
  const int maxp = pairs_per_dev[dev & 63];
  if (maxp <= 0) return cudaErrorNotSupported;  // no cluster of two can be resident
  CUtensorMap mq, ms, mo;
  cudaError_t e = make_map_bf16_3d(&mq, q, 256, S, N, 64, rp256::TOK);
  if (e == cudaSuccess) e = make_map_bf16_3d(&ms, Sfr_hilo, 256, 256, 2 * N, 64, 128);
  if (e == cudaSuccess) e = make_map_bf16_3d(&mo, out, 256, S, N, 64, rp256::TOK);
  if (e != cudaSuccess) return e;
  const int npair = (int)(N < maxp ? N : maxp);
  e = launch_pairs(k_readout256_pair_tc, npair, rp256::THREADS, rp256::SMEM, st, mq, ms, mo, (int)N, S);
  count_launch();
  return e;
}

// ============================================================================
// Chains of the recurrence on tensor cores for D = 256 (steps a4/a5 as one
// sequential chain per head, or one chain per reset block).
//
// Rows of the state are independent under X <- alpha (X - X Y) + Z, so each
// chain runs as two CTAs, one per 128-row half h of the 256 x 256 state. Per
// step one thread issues, over 16 slices of 16 k-rows,
//     P = X_hi Y_hi + X_lo Y_hi + X_hi Y_lo     (M = 128, N = 256, fp32 in TMEM)
// with X (this half's rows, K = 256) as a K-major bf16 (hi, lo) tile in shared
// memory and Y = A_t streaming in slices of its operand image through a
// 6-slot ring (one bulk copy per slice; the next frame's image and U_t rows
// are prefetched into L2 a step ahead). The fp32 state itself stays in TMEM
// next to P (columns 256..511). Eight epilogue warps read P and X, apply
// X <- gamma (X - P) + U_t with U_t read from global memory (L2), write X
// back to TMEM and, as a bf16 (hi, lo) pair, into the operand tile, which one
// thread then stores by TMA as the frame's state for the readout. U_t comes
// transposed from the contraction, so those reads coalesce.
//
// Operand image of a 256 x 256 matrix M (written by the contraction): 16
// slices of 16 rows k; slice s holds bf16(M) then bf16(M - bf16(M)) for rows
// 16s..16s+15, each as four 64-column blocks of [16 rows][128 B] in the
// 128-byte swizzled layout (block stride 2 KiB): 16 KiB per slice, 256 KiB in
// all (the size of the fp32 matrix).
// ============================================================================
namespace ch2 {
constexpr int D = 256;
constexpr int ATOM = 128 * 128;      // [128 rows][128 B]
constexpr int XT = 4 * ATOM;         // X hi (or lo) tile, K = 256: 64 KiB
constexpr int SLICE = 16 * 1024;     // 16 k-rows of the image: hi 8 KiB + lo 8 KiB
constexpr int NSLICE = D / 16;
constexpr int NSY = 6;               // Y ring slots
constexpr int OFF_XH = 0;
constexpr int OFF_XL = OFF_XH + XT;
constexpr int OFF_Y = OFF_XL + XT;
constexpr int OFF_BAR = OFF_Y + NSY * SLICE;
constexpr int NBAR = 2 * NSY + 3;    // y_full, y_empty, p_full, x_ready, fin
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM = OFF_MISC + 16 + 1024;
static_assert(SMEM <= 232448, "D = 256 chain shared memory");
constexpr int EPI = 256;             // 8 epilogue warps
constexpr int THREADS = 64 + EPI;    // producer warp, MMA warp, epilogue
constexpr uint32_t TMEM_COLS = 512;  // P: columns 0..255, fp32 state: 256..511
constexpr size_t IMG = (size_t)D * D * 4;
}  // namespace ch2

// Byte offset of 16-byte chunk n8 (columns 8 n8 .. 8 n8 + 7) of row k in the
// hi half of a D = 256 operand image (the lo half is 8 KiB further).
__device__ __forceinline__ int img256_off(int k, int n8) {
  const int s = k >> 4, rs = k & 15;
  return s * ch2::SLICE + (n8 >> 3) * 2048 + rs * 128 + (((n8 & 7) ^ (rs & 7)) << 4);
}

__global__ void __launch_bounds__(ch2::THREADS, 1)
    k_chain256_tc(ChainArgs a, const __grid_constant__ CUtensorMap tmSfr) {
  using namespace ch2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_yf = sb + OFF_BAR;
  const uint32_t bar_ye = bar_yf + 8 * NSY;
  const uint32_t bar_p = bar_ye + 8 * NSY;
  const uint32_t bar_x = bar_p + 8;
  const uint32_t bar_fin = bar_x + 8;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  const int half = blockIdx.x & 1;
  const ChainProg g = chain_prog(a, blockIdx.x >> 1);
  const size_t DD = (size_t)D * D;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSY; ++s) {
      mbar_init(bar_yf + 8 * s, 1);
      mbar_init(bar_ye + 8 * s, 1);
    }
    mbar_init(bar_p, 1);
    mbar_init(bar_x, EPI / 32);
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---- producer: Y slices through the ring; L2 prefetch a step ahead ----
    if (lane == 0) {
      int gi = 0;
      bool ok = true;
      for (int s = 0; s < g.n && ok; ++s) {
        const ChainStep st = chain_step_at(a, g, s);
        if (s + 1 < g.n) {
          const ChainStep nx = chain_step_at(a, g, s + 1);
          prefetch_l2(nx.Y, (uint32_t)IMG);
          prefetch_l2(nx.Z, (uint32_t)IMG);
        }
        for (int sl = 0; sl < NSLICE; ++sl, ++gi) {
          const int slot = gi % NSY;
          const uint32_t u = (uint32_t)(gi / NSY);
          ok = mbar_wait(bar_ye + 8 * slot, (u & 1) ^ 1, abort_flag, &g_tc_status, 41);
          if (!ok) break;
          mbar_arrive_expect_tx(bar_yf + 8 * slot, SLICE);
          bulk_load(sb + OFF_Y + slot * SLICE, (const uint8_t*)st.Y + (size_t)sl * SLICE, SLICE,
                    bar_yf + 8 * slot);
        }
      }
      // drain (bounded, not cut short by an abort): copies in flight land
      volatile int keep_waiting = 0;
      for (int gg = (gi > NSY ? gi - NSY : 0); gg < gi; ++gg)
        mbar_wait(bar_yf + 8 * (gg % NSY), (uint32_t)(gg / NSY) & 1, &keep_waiting, &g_tc_status, 42);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256, false, true);
      int gi = 0;
      bool ok = true;
      for (int s = 0; s < g.n && ok; ++s) {
        ok = mbar_wait(bar_x, (uint32_t)s & 1, abort_flag, &g_tc_status, 43);
        if (!ok) break;
        tc_fence_after();
        for (int sl = 0; sl < NSLICE; ++sl, ++gi) {
          const int slot = gi % NSY;
          const uint32_t u = (uint32_t)(gi / NSY);
          ok = mbar_wait(bar_yf + 8 * slot, u & 1, abort_flag, &g_tc_status, 44);
          if (!ok) break;
          tc_fence_after();
          const uint32_t xo = (sl >> 2) * ATOM + (sl & 3) * 32;
          const uint64_t dxh = smem_desc_sw128(sb + OFF_XH + xo, 16, 1024);
          const uint64_t dxl = smem_desc_sw128(sb + OFF_XL + xo, 16, 1024);
          const uint32_t ya = sb + OFF_Y + slot * SLICE;
          const uint64_t dyh = smem_desc_sw128(ya, 2048, 1024);
          const uint64_t dyl = smem_desc_sw128(ya + SLICE / 2, 2048, 1024);
          mma_bf16(tmem, dxh, dyh, idesc, sl > 0 ? 1u : 0u);
          mma_bf16(tmem, dxl, dyh, idesc, 1u);
          mma_bf16(tmem, dxh, dyl, idesc, 1u);
          mma_commit(bar_ye + 8 * slot);
        }
        if (!ok) break;
        mma_commit(bar_p);
      }
      mma_commit(bar_fin);
      volatile int keep_waiting = 0;
      mbar_wait(bar_fin, 0, &keep_waiting, &g_tc_status, 45);
    }
    __syncwarp();
  } else {
    // ---- epilogue: 8 warps; warp quadrant q = rows 32q.., column half ch ----
    const int et = threadIdx.x - 64;
    const int q = warp & 3, ch = et >> 7;
    const int row = q * 32 + lane;            // row of this CTA's half
    const size_t grow = (size_t)half * 128 + row;  // row of the state
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
    const bool store_sfr = g.mode == CHAIN_SCAN;
    int nstore = 0;
    float zb[2][32];
    // Z = U_t stored transposed: element (grow, col) at Z[col * D + grow], so
    // the warp's 32 rows read 128 contiguous bytes per column
    auto load_z = [&](const float* Z, int c, float* z) {
      const float* src = Z + (size_t)(128 * ch + 32 * c) * D + grow;
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] = __ldg(src + (size_t)i * D);
    };
    // the X tile (bf16 hi, lo) for columns 128 ch + 32 c .. +31 of this row
    auto put_x = [&](const float* x, int c) {
      const int col = 128 * ch + 32 * c;
      const int at = col >> 6, c0 = (col & 63) >> 3;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 hi, lo;
        split_chunk(x + 8 * i, &hi, &lo);
        const int off = at * ATOM + row * 128 + (((c0 + i) ^ (row & 7)) << 4);
        *(uint4*)(smem + OFF_XH + off) = hi;
        *(uint4*)(smem + OFF_XL + off) = lo;
      }
    };
    // initial state: fp32 rows of g.init (or zeros) into TMEM and the tile
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float x[32];
      const float* src = g.init ? g.init + grow * D + 128 * ch + 32 * c : nullptr;
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float4 f = src ? __ldg((const float4*)(src + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
        x[i] = f.x; x[i + 1] = f.y; x[i + 2] = f.z; x[i + 3] = f.w;
      }
      uint32_t xu[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) xu[i] = __float_as_uint(x[i]);
      tmem_st32(tl + 256 + 128 * ch + 32 * c, xu);
      put_x(x, c);
    }
    tmem_wait_st();
    fence_proxy_async();
    tc_fence_before();
    warp_arrive(bar_x);
    if (g.n > 0) {
      const ChainStep st0 = chain_step_at(a, g, 0);
      load_z(st0.Z, 0, zb[0]);
      load_z(st0.Z, 1, zb[1]);
    }
    for (int s = 0; s < g.n; ++s) {
      const ChainStep st = chain_step_at(a, g, s);
      bool ok = true;
      if (lane == 0) ok = mbar_wait(bar_p, (uint32_t)s & 1, abort_flag, &g_tc_status, 46);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      // the previous state store has read the tile; all agree on leaving
      if (et == 0 && nstore > 0) bulk_wait_read0();
      if (named_bar_or(1, EPI, !ok || *abort_flag)) break;
      tc_fence_after();
      const bool last = store_sfr && (g.j0 + s == a.T - 1) && a.state_out;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float* z = zb[c & 1];
        uint32_t p[32], xr[32];
        tmem_ld32(tl + 128 * ch + 32 * c, p);
        tmem_ld32(tl + 256 + 128 * ch + 32 * c, xr);
        tmem_wait_ld();
        float x[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          x[i] = st.reset ? z[i] : st.alpha * (__uint_as_float(xr[i]) - __uint_as_float(p[i])) + z[i];
          xr[i] = __float_as_uint(x[i]);
        }
        tmem_st32(tl + 256 + 128 * ch + 32 * c, xr);
        put_x(x, c);
        if (last) {
          float* so = a.state_out + (size_t)g.bh * DD + grow * D + 128 * ch + 32 * c;
#pragma unroll
          for (int i = 0; i < 32; i += 4) *(float4*)(so + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
        }
        if (c < 2) load_z(st.Z, c + 2, z);
      }
      tmem_wait_st();
      fence_proxy_async();
      tc_fence_before();
      if (s + 1 < g.n) {
        const ChainStep nx = chain_step_at(a, g, s + 1);
        load_z(nx.Z, 0, zb[0]);
        load_z(nx.Z, 1, zb[1]);
      }
      named_bar_sync(1, EPI);
      if (et == 0 && store_sfr) {
        // the state after frame t (this half's rows), as a bf16 (hi, lo) pair
        const int pair = g.bh * a.T + st.t;
#pragma unroll
        for (int at = 0; at < 4; ++at) {
          tma_store_3d(&tmSfr, sb + OFF_XH + at * ATOM, 64 * at, 128 * half, 2 * pair);
          tma_store_3d(&tmSfr, sb + OFF_XL + at * ATOM, 64 * at, 128 * half, 2 * pair + 1);
        }
        bulk_commit();
        ++nstore;
      }
      warp_arrive(bar_x);
    }
    if (et == 0) bulk_wait0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

static cudaError_t tc_chain256(const ChainArgs& a, int nchains, cudaStream_t st) {
  if (a.D != 256 || !a.y_image || a.mode != CHAIN_SCAN || !a.sfr_hilo) return cudaErrorNotSupported;
  if (a.seg == SEG_CHUNKS && a.nseg > 1) return cudaErrorNotSupported;  // span starts need the prefix
  static DeviceOnce attr_once;
  const cudaError_t attr_status = once_per_device(attr_once, [&]() -> cudaError_t {
    cudaError_t e =
        cudaFuncSetAttribute(k_chain256_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, ch2::SMEM);
    return e;
  });
  if (attr_status != cudaSuccess) return attr_status;
  const long long frames = (long long)a.heads * a.T;
  CUtensorMap ms;
  cudaError_t e = make_map_bf16_3d(&ms, a.Sfr, 256, 256, 2 * (uint64_t)frames, 64, 128);
  if (e != cudaSuccess) return e;
  k_chain256_tc<<<2 * nchains, ch2::THREADS, ch2::SMEM, st>>>(a, ms);
  count_launch();
  return cudaGetLastError();
}

// ============================================================================
// Backward token gradients on tensor cores (D = 128, bf16).
//
// Per frame-head, per 128-token tile of K and V (TMA, 128-byte swizzle):
//   [P2 | P5] = K [dAs | G^T]   (M = 128 tokens, N = 256, K = 128 channels)
//   P3        = V G             (N = 128; G read as an MN-major operand)
// with dAs = dA + dA^T and G = dL/dS_t in one per-frame bf16 operand (64 KiB,
// written by the per-frame kernel) kept in shared memory for the frame. With
// k^ = c k (c = 1/sqrt(D S)), per token s:
//   dk_s = c beta_s (c P2_s + P3_s),  dv_s = c beta_s P5_s,
//   dbeta_s = k^_s . (c P2_s / 2 + P3_s).
// Eight epilogue warps (two per TMEM lane quadrant, one per 64-channel half)
// stage dk and dv as bf16 in the tile's own V and K buffers and one thread
// stores them by TMA; dbeta halves meet in shared memory.
// ============================================================================
namespace btk {
constexpr int D = 128;
constexpr int TOK = 128;
constexpr int BOX = TOK * 128;                   // [128 tokens][64 channels] bf16: 16 KiB
constexpr int KT = 2 * BOX;                      // one tensor's tile: 32 KiB
constexpr int NST = 2;                           // K/V stages (also the dk/dv staging)
constexpr int BIMG = 65536;                      // per-frame B operand
constexpr int OFF_B = 0;
constexpr int OFF_KV = OFF_B + BIMG;             // stage s: K at OFF_KV + 2 s KT, V at + KT
constexpr int OFF_BETA = OFF_KV + NST * 2 * KT;  // [NST][TOK] fp32
constexpr int OFF_RED = OFF_BETA + NST * TOK * 4;  // [2][TOK][2] fp32 dbeta halves
constexpr int OFF_BAR = OFF_RED + 2 * TOK * 2 * 4;
constexpr int NBAR = 2 * NST + 5;  // full, empty per stage; b_full, b_empty, acc_full, acc_empty, fin
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM = OFF_MISC + 16 + 1024;
static_assert(SMEM <= 232448, "backward token kernel shared memory");
constexpr int EPI = 256;
constexpr int THREADS = 64 + EPI;
constexpr uint32_t TMEM_COLS = 512;  // [P2 | P5]: columns 0..255, P3: 256..383
}  // namespace btk

__global__ void __launch_bounds__(btk::THREADS, 1)
    k_bwd_tok_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                 const float* __restrict__ beta, const uint8_t* __restrict__ bimg,
                 float* __restrict__ dbeta, int N, int S, float c) {
  using namespace btk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_full = sb + OFF_BAR;
  const uint32_t bar_empty = bar_full + 8 * NST;
  const uint32_t bar_bf = bar_empty + 8 * NST;
  const uint32_t bar_be = bar_bf + 8;
  const uint32_t bar_accf = bar_be + 8;
  const uint32_t bar_acce = bar_accf + 8;
  const uint32_t bar_fin = bar_acce + 8;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full + 8 * s, 33);  // expect_tx arrival + 32 lanes' beta copies
      mbar_init(bar_empty + 8 * s, 1);  // the tile's dk/dv store has read its staging
    }
    mbar_init(bar_bf, 1);
    mbar_init(bar_be, 1);
    mbar_init(bar_accf, 1);
    mbar_init(bar_acce, EPI / 32);
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int ntile = (S + TOK - 1) / TOK;
  const int my_count = (int)blockIdx.x < N ? (N - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp == 0) {
    // ---- producer: the frame's B operand, K and V tiles (TMA), beta ----
    int g = 0, nb = 0;
    bool ok = true;
    for (int i = 0; i < my_count && ok; ++i) {
      const int n = blockIdx.x + i * gridDim.x;
      if (lane == 0) {
        ok = mbar_wait(bar_be, ((uint32_t)i & 1) ^ 1, abort_flag, &g_tc_status, 61);
        if (ok) {
          mbar_arrive_expect_tx(bar_bf, BIMG);
          bulk_load(sb + OFF_B, bimg + (size_t)n * BIMG, BIMG, bar_bf);
          ++nb;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      for (int tl = 0; tl < ntile && ok; ++tl, ++g) {
        const int s = g % NST;
        const uint32_t u = (uint32_t)(g / NST);
        if (lane == 0) ok = mbar_wait(bar_empty + 8 * s, (u & 1) ^ 1, abort_flag, &g_tc_status, 62);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        const uint32_t kd = sb + OFF_KV + s * 2 * KT, vd = kd + KT;
        if (lane == 0) {
          mbar_arrive_expect_tx(bar_full + 8 * s, 2 * KT);
          tma_load_3d(kd, &tmK, bar_full + 8 * s, 0, tl * TOK, n);
          tma_load_3d(kd + BOX, &tmK, bar_full + 8 * s, 64, tl * TOK, n);
          tma_load_3d(vd, &tmV, bar_full + 8 * s, 0, tl * TOK, n);
          tma_load_3d(vd + BOX, &tmV, bar_full + 8 * s, 64, tl * TOK, n);
        }
        const uint32_t bsa = sb + OFF_BETA + s * TOK * 4;
#pragma unroll
        for (int r = lane; r < TOK; r += 32) {
          const int tok = tl * TOK + r;
          const bool in = tok < S;
          cp_async_4(bsa + r * 4, beta + (size_t)n * S + (in ? tok : 0), in ? 4u : 0u);
        }
        cp_async_arrive_noinc(bar_full + 8 * s);
      }
    }
    // drain (bounded, not cut short by an abort): copies in flight land
    if (lane == 0) {
      volatile int keep_waiting = 0;
      for (int gg = (g > NST ? g - NST : 0); gg < g; ++gg)
        mbar_wait(bar_full + 8 * (gg % NST), (uint32_t)(gg / NST) & 1, &keep_waiting, &g_tc_status, 63);
      if (nb > 0) mbar_wait(bar_bf, (uint32_t)(nb - 1) & 1, &keep_waiting, &g_tc_status, 64);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      constexpr uint32_t idesc_k = idesc_bf16_f32(128, 256, false, false);
      constexpr uint32_t idesc_g = idesc_bf16_f32(128, 128, false, true);
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_count && ok; ++i) {
        ok = mbar_wait(bar_bf, (uint32_t)i & 1, abort_flag, &g_tc_status, 65);
        if (!ok) break;
        tc_fence_after();
        for (int tl = 0; tl < ntile; ++tl, ++g) {
          const int s = g % NST;
          ok = mbar_wait(bar_full + 8 * s, (uint32_t)(g / NST) & 1, abort_flag, &g_tc_status, 66);
          if (ok) ok = mbar_wait(bar_acce, ((uint32_t)g & 1) ^ 1, abort_flag, &g_tc_status, 67);
          if (!ok) break;
          tc_fence_after();
          const uint32_t ka = sb + OFF_KV + s * 2 * KT, va = ka + KT;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * BOX + (kk & 3) * 32;
            const uint64_t dk = smem_desc_sw128(ka + off, 16, 1024);
            const uint64_t dv = smem_desc_sw128(va + off, 16, 1024);
            // [dAs ; G] rows, K-major: 256 rows per 64-channel block of 32 KiB
            const uint64_t db = smem_desc_sw128(sb + OFF_B + (kk >> 2) * 32768 + (kk & 3) * 32, 16, 1024);
            // G as MN-major: 16 rows of k, column blocks 32 KiB apart
            const uint64_t dg = smem_desc_sw128(sb + OFF_B + 16384 + kk * 2048, 32768, 1024);
            mma_bf16(tmem, dk, db, idesc_k, kk > 0 ? 1u : 0u);
            mma_bf16(tmem + 256, dv, dg, idesc_g, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_accf);
        }
        if (!ok) break;
        mma_commit(bar_be);  // the frame's B operand is free once these MMAs are done
      }
      mma_commit(bar_fin);
      volatile int keep_waiting = 0;
      mbar_wait(bar_fin, 0, &keep_waiting, &g_tc_status, 68);
    }
    __syncwarp();
  } else {
    // ---- epilogue: 8 warps; quadrant q = token rows 32q.., half h = channels 64h.. ----
    const int et = threadIdx.x - 64;
    const int q = warp & 3, h = et >> 7;
    const int row = q * 32 + lane;
    const uint32_t tl_addr = tmem + ((uint32_t)(q * 32) << 16);
    int g = 0;
    for (int i = 0; i < my_count; ++i) {
      const int n = blockIdx.x + i * gridDim.x;
      bool stop = false;
      for (int tl = 0; tl < ntile; ++tl, ++g) {
        const int s = g % NST;
        int ok = 1;
        if (lane == 0) ok = mbar_wait(bar_accf, (uint32_t)g & 1, abort_flag, &g_tc_status, 69);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (named_bar_or(1, EPI, !ok || *abort_flag)) {
          stop = true;
          break;
        }
        tc_fence_after();
        uint8_t* kt = smem + OFF_KV + s * 2 * KT;
        uint8_t* vt = kt + KT;
        const float bv = ((const float*)(smem + OFF_BETA))[s * TOK + row];
        // this thread's 64 key channels (bf16 pairs), read before the K buffer
        // becomes the dv staging
        uint32_t kw[32];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 x = *(const uint4*)(kt + h * BOX + row * 128 + ((ch ^ (row & 7)) << 4));
          kw[4 * ch] = x.x; kw[4 * ch + 1] = x.y; kw[4 * ch + 2] = x.z; kw[4 * ch + 3] = x.w;
        }
        named_bar_sync(1, EPI);
        float dbp = 0.f;
#pragma unroll
        for (int c32 = 0; c32 < 2; ++c32) {
          uint32_t p2[32], p5[32], p3[32];
          const uint32_t col = 64 * h + 32 * c32;
          tmem_ld32(tl_addr + col, p2);
          tmem_ld32(tl_addr + 128 + col, p5);
          tmem_ld32(tl_addr + 256 + col, p3);
          tmem_wait_ld();
          float dkv[32], dvv[32];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kw[(32 * c32 + j) >> 1]));
            const float a2 = c * __uint_as_float(p2[j]), b2 = c * __uint_as_float(p2[j + 1]);
            const float a3 = __uint_as_float(p3[j]), b3 = __uint_as_float(p3[j + 1]);
            dkv[j] = c * bv * (a2 + a3);
            dkv[j + 1] = c * bv * (b2 + b3);
            dvv[j] = c * bv * __uint_as_float(p5[j]);
            dvv[j + 1] = c * bv * __uint_as_float(p5[j + 1]);
            dbp = fmaf(c * kf.x, 0.5f * a2 + a3, dbp);
            dbp = fmaf(c * kf.y, 0.5f * b2 + b3, dbp);
          }
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int ch = 4 * c32 + m;  // 16-byte chunk of the 128-byte row of box h
            const int off = h * BOX + row * 128 + ((ch ^ (row & 7)) << 4);
            *(uint4*)(vt + off) = make_uint4(pack_bf16x2(dkv[8 * m], dkv[8 * m + 1]),
                                             pack_bf16x2(dkv[8 * m + 2], dkv[8 * m + 3]),
                                             pack_bf16x2(dkv[8 * m + 4], dkv[8 * m + 5]),
                                             pack_bf16x2(dkv[8 * m + 6], dkv[8 * m + 7]));
            *(uint4*)(kt + off) = make_uint4(pack_bf16x2(dvv[8 * m], dvv[8 * m + 1]),
                                             pack_bf16x2(dvv[8 * m + 2], dvv[8 * m + 3]),
                                             pack_bf16x2(dvv[8 * m + 4], dvv[8 * m + 5]),
                                             pack_bf16x2(dvv[8 * m + 6], dvv[8 * m + 7]));
          }
        }
        tc_fence_before();
        warp_arrive(bar_acce);
        float* red = (float*)(smem + OFF_RED) + (g & 1) * TOK * 2;
        red[row * 2 + h] = dbp;
        fence_proxy_async();
        named_bar_sync(1, EPI);
        const int tok = tl * TOK + row;
        if (h == 0 && tok < S) dbeta[(size_t)n * S + tok] = red[row * 2] + red[row * 2 + 1];
        if (et == 0) {
          // dk from the V buffer, dv from the K buffer (rows past S are clipped)
          tma_store_3d(&tmDK, smem_u32(vt), 0, tl * TOK, n);
          tma_store_3d(&tmDK, smem_u32(vt + BOX), 64, tl * TOK, n);
          tma_store_3d(&tmDV, smem_u32(kt), 0, tl * TOK, n);
          tma_store_3d(&tmDV, smem_u32(kt + BOX), 64, tl * TOK, n);
          bulk_commit();
          bulk_wait_read0();
          mbar_arrive(bar_empty + 8 * s);
        }
      }
      if (stop) break;
    }
    if (et == 0) bulk_wait0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

cudaError_t tc_bwd_tokens(const void* k, const void* v, const float* beta, const void* bimg,
                          void* dk, void* dv, float* dbeta, long long N, int S, float c,
                          cudaStream_t st) {
  CUtensorMap mk, mv, mdk, mdv;
  cudaError_t e = make_map_bf16_3d(&mk, k, 128, S, N, 64, btk::TOK);
  if (e == cudaSuccess) e = make_map_bf16_3d(&mv, v, 128, S, N, 64, btk::TOK);
  if (e == cudaSuccess) e = make_map_bf16_3d(&mdk, dk, 128, S, N, 64, btk::TOK);
  if (e == cudaSuccess) e = make_map_bf16_3d(&mdv, dv, 128, S, N, 64, btk::TOK);
  if (e != cudaSuccess) return e;
  static DeviceOnce attr_once;
  const cudaError_t attr_status = once_per_device(attr_once, [&]() -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(k_bwd_tok_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, btk::SMEM);
    return e;
  });
  if (attr_status != cudaSuccess) return attr_status;
  const int grid = (int)(N < num_sms() ? N : num_sms());
  k_bwd_tok_tc<<<grid, btk::THREADS, btk::SMEM, st>>>(mk, mv, mdk, mdv, beta,
                                                      (const uint8_t*)bimg, dbeta, (int)N, S, c);
  count_launch();
  return cudaGetLastError();
}

// ============================================================================
// Backward per-frame terms on tensor cores (D = 128).
//
// Per frame (scan position j): dM = S'^T G and dM^T = G^T S' as split
// products (hi/lo pairs of both, three MMAs per 16 rows: ~16-bit operands),
// with S' = the state entering frame j (the previous frame's stored state,
// state_in for the first frame, zeros after a reset) and G = dL/dS after
// frame j, both bf16 (hi, lo) tiles brought in by TMA. Four epilogue warps
// (row i of dM each) then write
//   dA + dA^T = -gamma (dM + dM^T)        (rows 0..127 of the token kernel's
//   G rounded to bf16                      operand; rows 128..255)
//   dgamma = <dM, I - A>                   (A_t from its operand image)
// The accumulators (dM | dM^T, 256 columns) are double-buffered in TMEM, so
// one frame's epilogue runs under the next frame's loads and MMAs.
// ============================================================================
namespace bfr {
constexpr int D = 128;
constexpr int BOX = 128 * 128;          // [128 rows][64 columns] bf16: 16 KiB
constexpr int MAT = 4 * BOX;            // hi (2 boxes) + lo (2 boxes): 64 KiB
constexpr int OFF_S = 0;                // S' (hi, lo)
constexpr int OFF_G = OFF_S + MAT;      // G (hi, lo)
constexpr int OFF_BAR = OFF_G + MAT;
constexpr int NBAR = 2 + 2 + 2 + 1;     // in_full, in_empty, acc_full[2], acc_empty[2], fin
constexpr int OFF_RED = OFF_BAR + 8 * (NBAR + 1);
constexpr int OFF_MISC = OFF_RED + 4 * 4;
constexpr int SMEM = OFF_MISC + 16 + 1024;
constexpr int THREADS = 64 + 128;
constexpr uint32_t TMEM_COLS = 512;
}  // namespace bfr

// Which hi/lo source holds S' of frame-head n: 0 = stored states (index
// prev), 1 = converted state_in (index bh), 2 = zeros.
struct FrameSrc {
  int kind, idx;
};
__device__ __forceinline__ FrameSrc frame_prev_src(int n, int T, int reverse, int seq_reset,
                                                   int block, int has_s0) {
  const int bh = n / T, t = n % T;
  const int j = reverse ? T - 1 - t : t;
  if (j == 0) return FrameSrc{has_s0 ? 1 : 2, has_s0 ? bh : 0};
  const int tp = frame_at(j - 1, T, reverse);
  if (seq_reset && (t / block) != (tp / block)) return FrameSrc{2, 0};
  return FrameSrc{0, bh * T + tp};
}

__global__ void __launch_bounds__(bfr::THREADS, 1)
    k_bwd_frame_tc(const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmS0,
                   const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmG,
                   const uint8_t* __restrict__ Aimg, const __nv_bfloat16* __restrict__ Ghilo,
                   const float* __restrict__ gamma, float* __restrict__ dgamma,
                   uint8_t* __restrict__ bimg, int N, int T, int reverse, int seq_reset, int block,
                   int has_s0) {
  using namespace bfr;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_inf = sb + OFF_BAR;
  const uint32_t bar_ine = bar_inf + 8;
  const uint32_t bar_accf = bar_ine + 8;
  const uint32_t bar_acce = bar_accf + 16;
  const uint32_t bar_fin = bar_acce + 16;
  uint32_t* tmem_holder = (uint32_t*)(smem + OFF_MISC);
  volatile int* abort_flag = (volatile int*)(smem + OFF_MISC + 4);
  if (threadIdx.x == 0) {
    mbar_init(bar_inf, 1);
    mbar_init(bar_ine, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf + 8 * b, 1);
      mbar_init(bar_acce + 8 * b, 4);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int my_count = (int)blockIdx.x < N ? (N - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp == 0) {
    if (lane == 0) {
      int nin = 0;
      for (int i = 0; i < my_count; ++i) {
        const int n = blockIdx.x + i * gridDim.x;
        if (!mbar_wait(bar_ine, ((uint32_t)i & 1) ^ 1, abort_flag, &g_tc_status, 71)) break;
        const FrameSrc src = frame_prev_src(n, T, reverse, seq_reset, block, has_s0);
        const CUtensorMap* ms = src.kind == 0 ? &tmS : src.kind == 1 ? &tmS0 : &tmZ;
        mbar_arrive_expect_tx(bar_inf, 2 * MAT);
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            tma_load_3d(sb + OFF_S + (2 * hl + x) * BOX, ms, bar_inf, 64 * x, 0, 2 * src.idx + hl);
            tma_load_3d(sb + OFF_G + (2 * hl + x) * BOX, &tmG, bar_inf, 64 * x, 0, 2 * n + hl);
          }
        ++nin;
      }
      volatile int keep_waiting = 0;
      if (nin > 0) mbar_wait(bar_inf, (uint32_t)(nin - 1) & 1, &keep_waiting, &g_tc_status, 72);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, true, true);
      for (int i = 0; i < my_count; ++i) {
        const int b = i & 1;
        if (!mbar_wait(bar_acce + 8 * b, ((uint32_t)(i >> 1) & 1) ^ 1, abort_flag, &g_tc_status, 73))
          break;
        if (!mbar_wait(bar_inf, (uint32_t)i & 1, abort_flag, &g_tc_status, 74)) break;
        tc_fence_after();
        const uint32_t d = tmem + b * 256;
        const uint32_t sh = sb + OFF_S, sl = sh + 2 * BOX, gh = sb + OFF_G, gl = gh + 2 * BOX;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // rows r = 16 kk ..: S'^T and G^T as MN-major A, G and S' as MN-major B
          const uint32_t o = kk * 2048;
          const uint64_t dsh = smem_desc_sw128(sh + o, BOX, 1024), dsl = smem_desc_sw128(sl + o, BOX, 1024);
          const uint64_t dgh = smem_desc_sw128(gh + o, BOX, 1024), dgl = smem_desc_sw128(gl + o, BOX, 1024);
          const uint32_t acc = kk > 0 ? 1u : 0u;
          mma_bf16(d, dsh, dgh, idesc, acc);          // dM = S'^T G
          mma_bf16(d, dsl, dgh, idesc, 1u);
          mma_bf16(d, dsh, dgl, idesc, 1u);
          mma_bf16(d + 128, dgh, dsh, idesc, acc);    // dM^T = G^T S'
          mma_bf16(d + 128, dgl, dsh, idesc, 1u);
          mma_bf16(d + 128, dgh, dsl, idesc, 1u);
        }
        mma_commit(bar_ine);
        mma_commit(bar_accf + 8 * b);
      }
      mma_commit(bar_fin);
      volatile int keep_waiting = 0;
      mbar_wait(bar_fin, 0, &keep_waiting, &g_tc_status, 75);
    }
    __syncwarp();
  } else {
    // ---- epilogue: row i of dM per thread ----
    const int q = warp & 3;
    const int i_row = q * 32 + lane;
    float* red = (float*)(smem + OFF_RED);
    for (int i = 0; i < my_count; ++i) {
      const int n = blockIdx.x + i * gridDim.x;
      const int b = i & 1;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(bar_accf + 8 * b, (uint32_t)(i >> 1) & 1, abort_flag, &g_tc_status, 76);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (named_bar_or(1, 128, !ok || *abort_flag)) break;
      tc_fence_after();
      const float g = gamma[n];
      const uint8_t* aimg = Aimg + (size_t)n * kImageBytes;
      uint8_t* bo = bimg + (size_t)n * 65536;
      float part = 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t m[32], mt[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + b * 256 + c0, m);
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + b * 256 + 128 + c0, mt);
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          // 8 columns j = c0 + 8 ch ..: A_t row i_row from the image (hi + lo)
          const int col = c0 + 8 * ch;
          const int ao = (col >> 6) * 16384 + i_row * 128 + ((((col & 63) >> 3) ^ (i_row & 7)) << 4);
          const uint4 ah = *(const uint4*)(aimg + ao), al = *(const uint4*)(aimg + 32768 + ao);
          const uint32_t ahw[4] = {ah.x, ah.y, ah.z, ah.w}, alw[4] = {al.x, al.y, al.z, al.w};
          float o[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 fh = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ahw[e]));
            const float2 fl = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&alw[e]));
            const float a0 = fh.x + fl.x, a1 = fh.y + fl.y;
            const int j0 = col + 2 * e;
            const float m0 = __uint_as_float(m[8 * ch + 2 * e]), m1 = __uint_as_float(m[8 * ch + 2 * e + 1]);
            part += m0 * ((j0 == i_row ? 1.f : 0.f) - a0) + m1 * ((j0 + 1 == i_row ? 1.f : 0.f) - a1);
            o[2 * e] = -g * (m0 + __uint_as_float(mt[8 * ch + 2 * e]));
            o[2 * e + 1] = -g * (m1 + __uint_as_float(mt[8 * ch + 2 * e + 1]));
          }
          const int bo_off = (col >> 6) * 32768 + i_row * 128 + ((((col & 63) >> 3) ^ (i_row & 7)) << 4);
          *(uint4*)(bo + bo_off) = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                             pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
        }
      }
      tc_fence_before();
      warp_arrive(bar_acce + 8 * b);
      // G row i_row (hi + lo, rounded) -> operand row 128 + i_row
      const __nv_bfloat16* gh = Ghilo + (size_t)n * 2 * D * D + (size_t)i_row * D;
      const int r = 128 + i_row;
#pragma unroll 2
      for (int col = 0; col < 128; col += 8) {
        const uint4 hv = *(const uint4*)(gh + col), lv = *(const uint4*)(gh + (size_t)D * D + col);
        const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w}, lw[4] = {lv.x, lv.y, lv.z, lv.w};
        uint32_t ow[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fh = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hw[e]));
          const float2 fl = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lw[e]));
          ow[e] = pack_bf16x2(fh.x + fl.x, fh.y + fl.y);
        }
        const int off = (col >> 6) * 32768 + r * 128 + ((((col & 63) >> 3) ^ (r & 7)) << 4);
        *(uint4*)(bo + off) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      }
      // dgamma: sum over the 128 rows
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (lane == 0) red[q] = part;
      named_bar_sync(1, 128);
      if (threadIdx.x == 64) dgamma[n] = red[0] + red[1] + red[2] + red[3];
      named_bar_sync(1, 128);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// fp32 states [heads][D][D] -> bf16 (hi, lo) pairs [heads][2][D][D].
__global__ void k_to_hilo(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, int D) {
  const size_t mat = (size_t)D * D;
  const float* m = src + (size_t)blockIdx.x * mat;
  __nv_bfloat16* o = dst + (size_t)blockIdx.x * 2 * mat;
  for (size_t e = threadIdx.x; e < mat; e += blockDim.x) {
    const float x = m[e];
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    o[e] = h;
    o[mat + e] = __float2bfloat16_rn(x - __bfloat162float(h));
  }
}

cudaError_t tc_bwd_frames(const void* Sfr_hilo, const float* state_in, void* s0_hilo,
                          const void* zero_hilo, const void* G_hilo, const void* A_img,
                          const float* gamma, float* dgamma, void* bimg, long long N, int heads,
                          int T, int reverse, int seq_reset, int block, cudaStream_t st) {
  CUtensorMap ms, ms0, mz, mg;
  cudaError_t e = make_map_bf16_3d(&ms, Sfr_hilo, 128, 128, 2 * (uint64_t)N, 64, 128);
  if (e == cudaSuccess && state_in) {
    k_to_hilo<<<heads, 256, 0, st>>>(state_in, (__nv_bfloat16*)s0_hilo, 128);
    count_launch();
    e = cudaGetLastError();
  }
  if (e == cudaSuccess)
    e = make_map_bf16_3d(&ms0, state_in ? s0_hilo : zero_hilo, 128, 128,
                         state_in ? 2 * (uint64_t)heads : 2, 64, 128);
  if (e == cudaSuccess) e = make_map_bf16_3d(&mz, zero_hilo, 128, 128, 2, 64, 128);
  if (e == cudaSuccess) e = make_map_bf16_3d(&mg, G_hilo, 128, 128, 2 * (uint64_t)N, 64, 128);
  if (e != cudaSuccess) return e;
  static DeviceOnce attr_once;
  const cudaError_t attr_status = once_per_device(attr_once, [&]() -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(k_bwd_frame_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, bfr::SMEM);
    return e;
  });
  if (attr_status != cudaSuccess) return attr_status;
  const int grid = (int)(N < num_sms() ? N : num_sms());
  k_bwd_frame_tc<<<grid, bfr::THREADS, bfr::SMEM, st>>>(
      ms, ms0, mz, mg, (const uint8_t*)A_img, (const __nv_bfloat16*)G_hilo, gamma, dgamma,
      (uint8_t*)bimg, (int)N, T, reverse, seq_reset, block, state_in ? 1 : 0);
  count_launch();
  return cudaGetLastError();
}

// ---- public entry points of the tensor-core kernels (dispatch on D) ----
cudaError_t tc_contract(const void* k, const void* v, const float* beta, float* A, float* U,
                        long long N, int S, int D, float cA, float cU, int a_image,
                        const ProArgs* pro, cudaStream_t st) {
  if (D == 256) {
    if (pro) return cudaErrorNotSupported;
    return tc_contract256(k, v, beta, A, U, N, S, cA, cU, a_image, st);
  }
  if (D == 64) {
    if (pro) return cudaErrorNotSupported;
    CUtensorMap mk, mv;
    cudaError_t e = make_map_bf16_3d(&mk, k, 64, S, N, 64, c64::TOK);
    if (e != cudaSuccess) return e;
    e = make_map_bf16_3d(&mv, v, 64, S, N, 64, c64::TOK);
    if (e != cudaSuccess) return e;
    static DeviceOnce attr64_once;
    const cudaError_t attr_status = once_per_device(attr64_once, [&]() -> cudaError_t {
      cudaError_t e = cudaFuncSetAttribute(k_contract64_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, c64::SMEM);
      return e;
    });
    if (attr_status != cudaSuccess) return attr_status;
    const int grid = (int)(N < num_sms() ? N : num_sms());
    k_contract64_tc<<<grid, c64::THREADS, c64::SMEM, st>>>(mk, mv, beta, A, U, (int)N, S, cA, cU,
                                                            a_image);
    count_launch();
    return cudaGetLastError();
  }
  return tc_contract128(k, v, beta, A, U, N, S, D, cA, cU, a_image, pro, st);
}

cudaError_t tc_readout(const void* q, const void* Sfr_hilo, void* out, long long N, int S, int D,
                       const ProArgs* pro, cudaStream_t st) {
  if (D == 256) {
    if (pro) return cudaErrorNotSupported;
    return tc_readout256(q, Sfr_hilo, out, N, S, st);
  }
  if (D == 64) {
    if (pro) return cudaErrorNotSupported;
    CUtensorMap mq, ms, mo;
    cudaError_t e = make_map_bf16_3d(&mq, q, 64, S, N, 64, r64::TOK);
    if (e != cudaSuccess) return e;
    e = make_map_bf16_3d(&ms, Sfr_hilo, 64, 64, 2 * N, 64, 64);
    if (e != cudaSuccess) return e;
    e = make_map_bf16_3d(&mo, out, 64, S, N, 64, r64::TOK);
    if (e != cudaSuccess) return e;
    static DeviceOnce attr64_once;
    const cudaError_t attr_status = once_per_device(attr64_once, [&]() -> cudaError_t {
      cudaError_t e = cudaFuncSetAttribute(k_readout64_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, r64::SMEM);
      return e;
    });
    if (attr_status != cudaSuccess) return attr_status;
    const int parts = readout_parts(N, (S + r64::TOK - 1) / r64::TOK);
    const long long units = N * parts;
    const int grid = (int)(units < num_sms() ? units : num_sms());
    k_readout64_tc<<<grid, r64::THREADS, r64::SMEM, st>>>(mq, ms, mo, (int)N, S, parts);
    count_launch();
    return cudaGetLastError();
  }
  return tc_readout128(q, Sfr_hilo, out, N, S, D, pro, st);
}

cudaError_t tc_chain(const ChainArgs& a, int nchains, cudaStream_t st) {
  if (a.D == 64 && a.y_image) return tc_chain64(a, nchains, st);
  if (a.D == 256) return tc_chain256(a, nchains, st);
  return tc_chain128(a, nchains, st);
}

// Failure-path self test: one block waits (bounded by limit_ns) on an mbarrier
// that completes only if `arrive`; a wait that runs out is recorded in the
// status word with code 99 and the kernel returns normally.
__global__ void k_selftest_wait(int arrive, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (arrive && threadIdx.x == 0) mbar_arrive(b);
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_limit(b, 0, &abort_flag, &g_tc_status, 99, limit_ns);
}

cudaError_t tc_selftest_wait(int arrive, long long limit_ns, cudaStream_t st) {
  k_selftest_wait<<<1, 32, 0, st>>>(arrive, (unsigned long long)limit_ns);
  count_launch();
  return cudaGetLastError();
}

cudaError_t tc_read_status(int* status, cudaStream_t st) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(status, g_tc_status, sizeof(int), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyToSymbolAsync(g_tc_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

}  // namespace gdn
