// gdn_frame_scan_fwd_static: the frame scan with no memory allocation.
//
// Some callers cannot allocate device memory when they call the scan:
//  - streaming loops that run one short block of frames per call and must not
//    pay for cudaMalloc / cudaFree, which can synchronise the whole device and
//    stall the other streams of the pipeline;
//  - hosts whose device memory is already fully reserved by their own pooling
//    allocator, where a raw cudaMalloc fails even though the pool has room;
//  - plugin or callback contexts that receive input and output pointers but
//    no workspace and are not allowed to allocate.
// For them this entry point keeps its scratch in one fixed array in device
// memory, defined below, instead of allocating it.
#include <mutex>

#include "gdn_internal.cuh"

namespace gdn {

// The scratch array. Every GPU that loads this library holds these bytes until
// the process exits. All calls share it: a call leaves its contents behind,
// and two calls whose work overlaps on the GPU (different streams, or
// different host threads without ordering) race on it. Calls issued in order
// on one stream are safe.
constexpr size_t kStaticScratchBytes = 32u << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ptr[kMaxDevices] = {};

// The device address of the array on the current device, looked up once per
// device (host code only sees a host-side stand-in for the symbol). The address
// stays valid for the life of the device's primary context; after a
// cudaDeviceReset the module may load elsewhere, so this entry point must not
// be used across a device reset.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    g_ptr[dev] = p;
  }
  *out = g_ptr[dev];
  return cudaSuccess;
}
}  // namespace

int scan_ex_entry(const gdn_params& p, cudaStream_t st);  // gdn_api.cu
int set_last_error(int status, const char* msg);          // gdn_api.cu

}  // namespace gdn

using namespace gdn;

extern "C" int gdn_frame_scan_fwd_static(const void* q, const void* k, const void* v,
                                         const float* beta, const float* gamma,
                                         const float* state_in, void* out, float* state_out,
                                         int B, int H, int T, int S, int D, unsigned flags,
                                         gdn_stream_t stream) {
  if (flags & (GDN_FUSED_PROLOGUE | GDN_BIDIR))
    return set_last_error(GDN_ERR_INVALID,
                          "gdn_frame_scan_fwd_static takes neither GDN_FUSED_PROLOGUE nor GDN_BIDIR");
  const size_t need = gdn_workspace_bytes(B, H, T, S, D, flags);
  if (need == 0) return set_last_error(GDN_ERR_INVALID, "invalid sizes");
  if (need > kStaticScratchBytes)
    return set_last_error(GDN_ERR_WORKSPACE,
                          "these sizes need more scratch than the fixed 32 MiB of "
                          "gdn_frame_scan_fwd_static; use gdn_frame_scan_fwd_ex");
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) return set_last_error(GDN_ERR_CUDA, cudaGetErrorString(e));
  gdn_params p = {};
  p.q = q;
  p.k = k;
  p.v = v;
  p.beta = beta;
  p.gamma = gamma;
  p.state_in = state_in;
  p.out = out;
  p.state_out = state_out;
  p.B = B;
  p.H = H;
  p.T = T;
  p.S = S;
  p.D = D;
  p.flags = flags;
  p.workspace = scratch;
  p.workspace_bytes = kStaticScratchBytes;
  return scan_ex_entry(p, (cudaStream_t)stream);
}
