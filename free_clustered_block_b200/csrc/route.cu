// Assignment: centroid scores and exact top-k per query cluster.
//
// ClusterAttention paper, Section 3.3.1 "Scoring": s_ab = qbar_a . kbar_b is
// exactly the mean logit between the two clusters (eq. 18); Section 3.3.2
// "Selection": each query cluster keeps its k best-scoring key clusters.
// Scores are fp64; the selection is exact, equal scores ordered by the lower
// key-cluster index, and the kept list is written in ascending order.
#include "ca_internal.cuh"

namespace ca {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kRouteTile = 64;   // key centroids staged per step

template <int D>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const double* __restrict__ qbar,
                                                              const double* __restrict__ kbar, int C,
                                                              int Cpad, int k, int32_t* __restrict__ kept_idx,
                                                              uint32_t* __restrict__ kept_bits) {
  constexpr int P = kRouteThreads / kRouteTile;   // partial sums per score
  constexpr int DP = D / P;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* qa = reinterpret_cast<double*>(smem_raw);        // D
  double* kt = qa + D;                                     // kRouteTile * (D + 1)
  double* part = kt + kRouteTile * (D + 1);                // kRouteThreads
  double* sc = part + kRouteThreads;                       // Cpad
  int* id = reinterpret_cast<int*>(sc + Cpad);             // Cpad
  uint32_t* bits = reinterpret_cast<uint32_t*>(id + Cpad); // Cpad / 32
  __shared__ int woff[kRouteThreads + 1];

  const int a = blockIdx.x, bh = blockIdx.y;
  const double* kb = kbar + (size_t)bh * C * D;
  if (threadIdx.x < D) qa[threadIdx.x] = qbar[((size_t)bh * C + a) * D + threadIdx.x];
  const int bl = threadIdx.x % kRouteTile, pp = threadIdx.x / kRouteTile;
  for (int b0 = 0; b0 < Cpad; b0 += kRouteTile) {
    __syncthreads();
    for (int e = threadIdx.x; e < kRouteTile * D; e += kRouteThreads) {
      const int r = e / D, col = e % D, b = b0 + r;
      kt[r * (D + 1) + col] = (b < C) ? kb[(size_t)b * D + col] : 0.0;
    }
    __syncthreads();
    double s = 0.0;
#pragma unroll 8
    for (int j = pp * DP; j < (pp + 1) * DP; ++j) s = fma(qa[j], kt[bl * (D + 1) + j], s);
    part[threadIdx.x] = s;
    __syncthreads();
    if (threadIdx.x < kRouteTile) {
      const int b = b0 + threadIdx.x;
      double t = 0.0;
      for (int q = 0; q < P; ++q) t += part[q * kRouteTile + threadIdx.x];
      sc[b] = (b < C) ? t : -INFINITY;
      id[b] = (b < C) ? b : 0x7fffffff;
    }
  }
  __syncthreads();
  // Bitonic sort: descending score, ascending index.
  for (int size = 2; size <= Cpad; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < Cpad; i += kRouteThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const double si = sc[i], sj = sc[j];
          const int ii = id[i], ij = id[j];
          const bool i_first = (si > sj) || (si == sj && ii < ij);
          const bool up = ((i & size) == 0);
          if (up ? !i_first : i_first) { sc[i] = sj; sc[j] = si; id[i] = ij; id[j] = ii; }
        }
      }
      __syncthreads();
    }
  }
  const int W = (C + 31) / 32;
  for (int w = threadIdx.x; w < W; w += kRouteThreads) bits[w] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < k; i += kRouteThreads) atomicOr(&bits[id[i] >> 5], 1u << (id[i] & 31));
  __syncthreads();
  uint32_t* brow = kept_bits + ((size_t)bh * C + a) * W;
  for (int w = threadIdx.x; w < W; w += kRouteThreads) brow[w] = bits[w];
  // Ascending kept list from the bitmask (W <= 256 words per pass).
  int32_t* krow = kept_idx + ((size_t)bh * C + a) * k;
  for (int w0 = 0, base = 0; w0 < W; w0 += kRouteThreads) {
    const int w = w0 + threadIdx.x;
    const int pc = (w < W) ? __popc(bits[w]) : 0;
    if (threadIdx.x == 0) woff[0] = 0;
    __syncthreads();
    // serial exclusive scan (W is small)
    if (threadIdx.x == 0) {
      int s = 0;
      for (int i = 0; i < kRouteThreads; ++i) {
        const int ww = w0 + i;
        woff[i] = s;
        s += (ww < W) ? __popc(bits[ww]) : 0;
      }
      woff[kRouteThreads] = s;
    }
    __syncthreads();
    if (w < W) {
      uint32_t m = bits[w];
      int o = base + woff[threadIdx.x];
      while (m) {
        const int bpos = __ffs(m) - 1;
        krow[o++] = w * 32 + bpos;
        m &= m - 1;
      }
    }
    (void)pc;
    base += woff[kRouteThreads];
    __syncthreads();
  }
}

}  // namespace

size_t route_smem_bytes(int C, int D) {
  int Cpad = 1;
  while (Cpad < C) Cpad <<= 1;
  if (Cpad < kRouteTile) Cpad = kRouteTile;
  return (size_t)D * 8 + (size_t)kRouteTile * (D + 1) * 8 + kRouteThreads * 8 + (size_t)Cpad * 12 +
         (size_t)(Cpad / 32 + 1) * 4;
}

cudaError_t launch_route(const ca_shape* s, int C, const double* qbar, const double* kbar, int k,
                         int32_t* kept_idx, uint32_t* kept_bits, cudaStream_t st) {
  int Cpad = 1;
  while (Cpad < C) Cpad <<= 1;
  if (Cpad < kRouteTile) Cpad = kRouteTile;
  const size_t smem = route_smem_bytes(C, s->d);
  const dim3 grid(C, s->B * s->H);
  if (s->d == 64) {
    cudaFuncSetAttribute(route_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    route_kernel<64><<<grid, kRouteThreads, smem, st>>>(qbar, kbar, C, Cpad, k, kept_idx, kept_bits);
  } else {
    cudaFuncSetAttribute(route_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    route_kernel<128><<<grid, kRouteThreads, smem, st>>>(qbar, kbar, C, Cpad, k, kept_idx, kept_bits);
  }
  return cudaGetLastError();
}

}  // namespace ca
