// gdn_frame_scan_fwd_host: the frame scan over buffers in HOST memory.
//
// Heads are independent, so the call streams them through the GPU in chunks
// of whole heads: while chunk c is scanned, chunk c+1 is copied in and chunk
// c-1 copied out, on three CUDA streams, so that PCIe carries both
// directions at once and the scans hide under the copies. Two device slots
// (inputs, outputs and scan workspace for one chunk each) alternate; events
// order each slot's reuse. One cudaMemcpyAsync per tensor and chunk.
#include <stdio.h>
#include <string.h>

#include "gdn_internal.cuh"

namespace gdn {
int scan_ex_entry(const gdn_params& p, cudaStream_t st);  // gdn_api.cu
int set_last_error(int status, const char* msg);          // gdn_api.cu
}  // namespace gdn

using namespace gdn;

namespace {

struct Slot {
  char* q = nullptr;
  char* k = nullptr;
  char* v = nullptr;
  float* beta = nullptr;
  float* gamma = nullptr;
  float* s_in = nullptr;
  char* out = nullptr;
  float* s_out = nullptr;
  void* ws = nullptr;
};

struct Pipeline {
  cudaStream_t st[3] = {nullptr, nullptr, nullptr};  // copies in, scans, copies out
  cudaEvent_t ev[3][2] = {};                         // per stream and slot
  void* block = nullptr;                             // one allocation for both slots
  cudaStream_t owner = nullptr;

  ~Pipeline() {
    for (cudaStream_t s : st)
      if (s) cudaStreamSynchronize(s);
    if (block) cudaFreeAsync(block, owner);
    if (owner) cudaStreamSynchronize(owner);
    for (auto& row : ev)
      for (cudaEvent_t e : row)
        if (e) cudaEventDestroy(e);
    for (cudaStream_t s : st)
      if (s) cudaStreamDestroy(s);
  }
};

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

int fail_cuda(cudaError_t e, const char* where) {
  char buf[256];
  snprintf(buf, sizeof(buf), "gdn_frame_scan_fwd_host: %s: %s", where, cudaGetErrorString(e));
  return set_last_error(GDN_ERR_CUDA, buf);
}

}  // namespace

extern "C" int gdn_frame_scan_fwd_host(const void* q, const void* k, const void* v,
                                       const float* beta, const float* gamma,
                                       const float* state_in, void* out, float* state_out, int B,
                                       int H, int T, int S, int D, unsigned flags,
                                       int heads_per_chunk, gdn_stream_t stream) {
  set_last_error(GDN_OK, "");
  if (flags & (GDN_FUSED_PROLOGUE | GDN_BIDIR | GDN_UCPE))
    return set_last_error(GDN_ERR_INVALID,
                          "gdn_frame_scan_fwd_host takes the flags of gdn_frame_scan_fwd");
  if (B < 1 || H < 1 || T < 1 || S < 1 || D < 1)
    return set_last_error(GDN_ERR_INVALID, "sizes must be >= 1");
  if (!q || !k || !v || !beta || !gamma || !out)
    return set_last_error(GDN_ERR_INVALID, "null q/k/v/beta/gamma/out");
  if (heads_per_chunk < 0) return set_last_error(GDN_ERR_INVALID, "heads_per_chunk must be >= 0");
  const long long heads = (long long)B * H;
  const int hc = (int)(heads_per_chunk == 0 ? (heads < 2 ? heads : 2)
                                            : (heads_per_chunk < heads ? heads_per_chunk : heads));
  const size_t elt = (flags & GDN_BF16) ? 2 : 4;
  const size_t tens_h = (size_t)T * S * D * elt;  // one head of q, k, v or out
  const size_t beta_h = (size_t)T * S * 4, gamma_h = (size_t)T * 4, mat_h = (size_t)D * D * 4;
  const size_t ws_bytes = gdn_workspace_bytes(1, hc, T, S, D, flags);
  if (ws_bytes == 0) return set_last_error(GDN_ERR_UNSUPPORTED, "unsupported sizes");

  // slot layout: q, k, v, out, beta, gamma, state_in, state_out, workspace
  const size_t o_q = 0, o_k = up256(o_q + hc * tens_h), o_v = up256(o_k + hc * tens_h),
               o_out = up256(o_v + hc * tens_h), o_beta = up256(o_out + hc * tens_h),
               o_gamma = up256(o_beta + hc * beta_h), o_sin = up256(o_gamma + hc * gamma_h),
               o_sout = up256(o_sin + hc * mat_h), o_ws = up256(o_sout + hc * mat_h),
               slot_bytes = up256(o_ws + ws_bytes);

  Pipeline pl;
  pl.owner = (cudaStream_t)stream;
  cudaError_t e = cudaMallocAsync(&pl.block, 2 * slot_bytes, pl.owner);
  if (e != cudaSuccess) return fail_cuda(e, "device slots");
  cudaEvent_t ready = nullptr;
  e = cudaEventCreateWithFlags(&ready, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventRecord(ready, pl.owner);
  for (int i = 0; i < 3 && e == cudaSuccess; ++i) {
    e = cudaStreamCreateWithFlags(&pl.st[i], cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(pl.st[i], ready, 0);  // after prior work and the allocation
    for (int j = 0; j < 2 && e == cudaSuccess; ++j)
      e = cudaEventCreateWithFlags(&pl.ev[i][j], cudaEventDisableTiming);
  }
  if (ready) cudaEventDestroy(ready);
  if (e != cudaSuccess) return fail_cuda(e, "streams");

  Slot slot[2];
  for (int j = 0; j < 2; ++j) {
    char* b = (char*)pl.block + j * slot_bytes;
    slot[j].q = b + o_q;
    slot[j].k = b + o_k;
    slot[j].v = b + o_v;
    slot[j].out = b + o_out;
    slot[j].beta = (float*)(b + o_beta);
    slot[j].gamma = (float*)(b + o_gamma);
    slot[j].s_in = (float*)(b + o_sin);
    slot[j].s_out = (float*)(b + o_sout);
    slot[j].ws = b + o_ws;
  }
  cudaStream_t s_in = pl.st[0], s_cmp = pl.st[1], s_out = pl.st[2];
  bool used[2] = {false, false};
  const cudaMemcpyKind H2D = cudaMemcpyHostToDevice, D2H = cudaMemcpyDeviceToHost;
  for (long long h0 = 0, c = 0; h0 < heads; h0 += hc, ++c) {
    const int n = (int)(heads - h0 < hc ? heads - h0 : hc);
    const int j = (int)(c & 1);
    Slot& sl = slot[j];
    // copies in: the slot's previous scan must have read it
    if (used[j]) e = cudaStreamWaitEvent(s_in, pl.ev[1][j], 0);
    const struct {
      void* dst;
      const void* src;
      size_t per_head;
    } ins[] = {{sl.q, q, tens_h},           {sl.k, k, tens_h},         {sl.v, v, tens_h},
               {sl.beta, beta, beta_h},     {sl.gamma, gamma, gamma_h}, {sl.s_in, state_in, mat_h}};
    for (const auto& x : ins) {
      if (e != cudaSuccess || !x.src) continue;
      e = cudaMemcpyAsync(x.dst, (const char*)x.src + h0 * x.per_head, n * x.per_head, H2D, s_in);
    }
    if (e == cudaSuccess) e = cudaEventRecord(pl.ev[0][j], s_in);
    // the scan: after its inputs, and after the slot's previous outputs left
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_cmp, pl.ev[0][j], 0);
    if (e == cudaSuccess && used[j]) e = cudaStreamWaitEvent(s_cmp, pl.ev[2][j], 0);
    if (e != cudaSuccess) return fail_cuda(e, "copies in");
    gdn_params p;
    memset(&p, 0, sizeof(p));
    p.q = sl.q;
    p.k = sl.k;
    p.v = sl.v;
    p.beta = sl.beta;
    p.gamma = sl.gamma;
    p.state_in = state_in ? sl.s_in : nullptr;
    p.out = sl.out;
    p.state_out = sl.s_out;
    p.B = 1;
    p.H = n;
    p.T = T;
    p.S = S;
    p.D = D;
    p.flags = flags;
    p.workspace = sl.ws;
    p.workspace_bytes = ws_bytes;
    const int rc = scan_ex_entry(p, s_cmp);
    if (rc != GDN_OK) return rc;  // its message is already set
    e = cudaEventRecord(pl.ev[1][j], s_cmp);
    // copies out
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, pl.ev[1][j], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync((char*)out + h0 * tens_h, sl.out, n * tens_h, D2H, s_out);
    if (e == cudaSuccess && state_out)
      e = cudaMemcpyAsync((char*)state_out + h0 * mat_h, sl.s_out, n * mat_h, D2H, s_out);
    if (e == cudaSuccess) e = cudaEventRecord(pl.ev[2][j], s_out);
    if (e != cudaSuccess) return fail_cuda(e, "copies out");
    used[j] = true;
  }
  // the results are in host memory when the call returns
  for (cudaStream_t s : pl.st) {
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail_cuda(e, "synchronize");
  }
  return GDN_OK;
}
