// Tensor-core (tcgen05) block-sparse attention: placeholder that routes to
// the CUDA-core kernel until the sm_100a kernel lands.
#include "ca_internal.cuh"

namespace ca {

__device__ unsigned int g_device_error = 0;
static uint64_t g_wait_limit = 0;
constexpr uint64_t kDefaultWaitLimit = 1ull << 26;

uint64_t wait_limit() { return g_wait_limit ? g_wait_limit : kDefaultWaitLimit; }
void set_wait_limit(uint64_t spins) { g_wait_limit = spins; }

cudaError_t device_error_read_clear(unsigned* out, cudaStream_t st) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_device_error, sizeof(unsigned), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  const unsigned zero = 0;
  e = cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(unsigned), 0, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

cudaError_t launch_attend_tc(const ca_shape* s, const ca_clusters* cl, const ca_routes* rt, int compensate,
                             void* O, const AttendWs& L, char* ws, cudaStream_t st) {
  return cudaErrorNotSupported;
}

cudaError_t launch_dense_tc(const void* Q, const void* K, const void* V, const ca_shape* s, void* O,
                            cudaStream_t st) {
  return launch_dense_simt(Q, K, V, s, O, st);
}

}  // namespace ca
