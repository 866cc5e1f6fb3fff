// Tensor-core (tcgen05) kernels: placeholder until the sm_100a kernels land.
#include "gdn_internal.cuh"

namespace gdn {

static __device__ int g_tc_status = 0;

bool tc_contract_supported(int) { return false; }
bool tc_readout_supported(int) { return false; }
bool tc_chain_supported(int) { return false; }
cudaError_t tc_contract(const void*, const void*, const float*, float*, float*, long long, int,
                        int, float, float, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t tc_readout(const void*, const void*, void*, long long, int, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t tc_chain(const ChainArgs&, int, cudaStream_t) { return cudaErrorNotSupported; }

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
