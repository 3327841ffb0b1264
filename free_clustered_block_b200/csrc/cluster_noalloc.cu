// ca_cluster without a caller-provided workspace.
//
// Some callers cannot hand this library device memory: code that runs as a
// plugin inside another framework that owns every device allocation and
// offers no scratch buffer, and latency-critical loops that must never call
// cudaMalloc (it can synchronise the device and can fail in the middle of a
// run). For them the clustering scratch lives in a fixed array in device
// global memory that belongs to this library.
#include <cuda.h>

#include <mutex>

#include "ca_internal.cuh"

namespace {

// Stated maximum: 16 MiB of scratch, enough for e.g. two 65,536-token heads
// at d = 64 or one 75,600-token head at d = 128 (ca_cluster_workspace_bytes
// gives the need of a shape).
constexpr size_t kScratchBytes = 16ull << 20;

// Every GPU on which this module is loaded holds these 16 MiB until the
// process exits.
__device__ __align__(256) unsigned char g_cluster_scratch[kScratchBytes];

// Device address of g_cluster_scratch per device ordinal, with the context
// it was looked up in. In host code the symbol's name is only a host-side
// stand-in, so the address is looked up with cudaGetSymbolAddress, once per
// device, with that device current. The module (and with it the array) is
// loaded again when the device's primary context is destroyed and re-created
// (cudaDeviceReset), so the cached address is used only while the current
// context is the one it was looked up in; otherwise it is looked up afresh.
constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
CUcontext g_scratch_ctx[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
  }
  return fn;
}

}  // namespace

extern "C" ca_status ca_cluster_noalloc(const void* Q, const void* K, const ca_shape* shape,
                                        const ca_cluster_params* params, const ca_clusters* out,
                                        void* stream) {
  ca_status st = ca_check_shape(shape);
  if (st != CA_OK) return st;
  const size_t need = ca_cluster_workspace_bytes(shape);
  if (need == 0) return CA_ERR_UNSUPPORTED;
  if (need > kScratchBytes) return CA_ERR_WORKSPACE;   // shape too large for the fixed scratch
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return CA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    // cudaGetSymbolAddress makes the device's primary context current first,
    // so look the address up before reading which context is current.
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_cluster_scratch) != cudaSuccess || p == nullptr) return CA_ERR_CUDA;
      g_scratch_addr[dev] = p;
      g_scratch_ctx[dev] = nullptr;
    }
    CtxGetCurrentFn get = ctx_get_current();
    CUcontext ctx = nullptr;
    if (!get || get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return CA_ERR_CUDA;
    if (g_scratch_ctx[dev] == nullptr) {
      g_scratch_ctx[dev] = ctx;
    } else if (g_scratch_ctx[dev] != ctx) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_cluster_scratch) != cudaSuccess || p == nullptr) return CA_ERR_CUDA;
      g_scratch_addr[dev] = p;
      g_scratch_ctx[dev] = ctx;
    }
    scratch = g_scratch_addr[dev];
  }
  // Every scratch byte the clustering kernels read is written earlier in the
  // same call, so the previous call's contents need no clearing.
  return ca_cluster(Q, K, shape, params, out, scratch, kScratchBytes, stream);
}
