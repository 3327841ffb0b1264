// Assignment: centroid scores and exact top-k per query cluster.
//
// ClusterAttention paper, Section 3.3.1 "Scoring": s_ab = qbar_a . kbar_b is
// exactly the mean logit between the two clusters (eq. 18); Section 3.3.2
// "Selection": each query cluster keeps its k best-scoring key clusters.
// Scores are fp64; the selection is exact, equal scores ordered by the lower
// key-cluster index, and the kept list is written in ascending order.
//
// A block handles QA query clusters of one head.
//  * Scores: thread t holds key centroid b = t, t + 256, ... in registers (64
//    columns at a time) and forms its QA dot products against the query
//    centroids, which every lane reads from shared memory as broadcasts. The
//    dot product runs over the columns in order with one fma chain.
//  * Selection: one warp per query cluster runs a radix select over the
//    order-preserving 64-bit keys of the scores, 8 bits per pass from the top,
//    starting below the prefix that all C keys share. A pass histograms the
//    keys that still match the decided prefix and picks the digit where the
//    running count from the top reaches the number still to take; it stops as
//    soon as that whole digit bin is taken. Keys above the final prefix are
//    kept; keys equal to it are kept in ascending index order until k are
//    kept. The kept bitmask word w is the warp's ballot over keys 32w..32w+31.
#include "ca_internal.cuh"

namespace ca {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / 32;
// one block per SM either way (its registers), so the score rows may use most of shared memory
constexpr size_t kRouteSmemBudget = 200 * 1024;

// C query clusters (rows), Ck key clusters (columns).
template <int D, int QA>
__global__ void __launch_bounds__(kRouteThreads, 1) route_kernel(const double* __restrict__ qbar,
                                                                 const double* __restrict__ kbar, int C, int Ck, int k,
                                                                 int32_t* __restrict__ kept_idx,
                                                                 uint32_t* __restrict__ kept_bits,
                                                                 int32_t* __restrict__ kept_count) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* qs = reinterpret_cast<double*>(smem_raw);   // QA x D
  double* sc = qs + QA * D;                           // QA x Ck scores
  __shared__ uint32_t hist[kRouteWarps][256];

  const int a0 = blockIdx.x * QA, bh = blockIdx.y;
  const int nq = min(QA, C - a0);
  for (int e = threadIdx.x; e < QA * D; e += kRouteThreads) {
    const int r = e / D;
    qs[e] = r < nq ? qbar[((size_t)bh * C + a0 + r) * D + (e % D)] : 0.0;
  }
  __syncthreads();

  // ---- scores ----
  const double* kb = kbar + (size_t)bh * Ck * D;
  for (int b = threadIdx.x; b < Ck; b += kRouteThreads) {
    double s[QA];
#pragma unroll
    for (int r = 0; r < QA; ++r) s[r] = 0.0;
#pragma unroll
    for (int h = 0; h < D; h += 64) {
      double kr[64];
      const double2* src = reinterpret_cast<const double2*>(kb + (size_t)b * D + h);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const double2 v = __ldg(src + i);
        kr[2 * i] = v.x; kr[2 * i + 1] = v.y;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
#pragma unroll
        for (int r = 0; r < QA; ++r) {
          const double2 q2 = *reinterpret_cast<const double2*>(qs + r * D + h + 2 * i);
          s[r] = fma(q2.x, kr[2 * i], s[r]);
          s[r] = fma(q2.y, kr[2 * i + 1], s[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < QA; ++r) sc[(size_t)r * Ck + b] = s[r];
  }
  __syncthreads();

  // ---- selection, one warp per query cluster ----
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  const int W = (Ck + 31) / 32;
  uint32_t* h = hist[warp];
  for (int r = warp; r < nq; r += kRouteWarps) {
    const double* row = sc + (size_t)r * Ck;
    // common prefix of all keys
    uint64_t kand = ~0ull, kor = 0ull;
    for (int b = lane; b < Ck; b += 32) {
      const uint64_t key = ordered_key(row[b]);
      kand &= key; kor |= key;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      kand &= __shfl_xor_sync(0xffffffffu, kand, o);
      kor |= __shfl_xor_sync(0xffffffffu, kor, o);
    }
    const uint64_t diff = kand ^ kor;
    int L = diff ? (__clzll((long long)diff) & ~7) : 64;   // decided prefix length (bits)
    uint64_t P = L == 0 ? 0ull : (L == 64 ? kand : kand >> (64 - L));
    int krem = k;                     // still to take among keys whose prefix equals P
    bool all = (k >= Ck);             // every key matching P is kept
    while (!all && L < 64) {
      for (int i = lane; i < 256; i += 32) h[i] = 0u;
      __syncwarp();
      const int shift = 56 - L;
      for (int b0 = 0; b0 < Ck; b0 += 32) {
        const int b = b0 + lane;
        int dig = 256 + lane;          // no bin
        if (b < Ck) {
          const uint64_t key = ordered_key(row[b]);
          if (L == 0 || (key >> (64 - L)) == P) dig = (int)((key >> shift) & 255u);
        }
        const unsigned grp = __match_any_sync(0xffffffffu, dig);
        if (dig < 256 && (grp & lt) == 0u) atomicAdd(&h[dig], (uint32_t)__popc(grp));
      }
      __syncwarp();
      // lane l owns bins 255 - 8l ... 248 - 8l, scanned from the top
      uint32_t cnt[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { cnt[j] = h[255 - 8 * lane - j]; tot += cnt[j]; }
      uint32_t inc = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
      }
      const uint32_t exc = inc - tot;
      const bool mine = exc < (uint32_t)krem && (uint32_t)krem <= inc;
      const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
      int dsel = 0;
      uint32_t above = 0, inbin = 0;
      if (mine) {
        uint32_t c = exc;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (inbin == 0u && c + cnt[j] >= (uint32_t)krem) { dsel = 255 - 8 * lane - j; above = c; inbin = cnt[j]; }
          c += cnt[j];
        }
      }
      dsel = __shfl_sync(0xffffffffu, dsel, src);
      above = __shfl_sync(0xffffffffu, above, src);
      inbin = __shfl_sync(0xffffffffu, inbin, src);
      krem -= (int)above;
      P = (P << 8) | (uint64_t)dsel;
      L += 8;
      if (inbin == (uint32_t)krem) all = true;
      __syncwarp();
    }
    // membership, bitmask and ascending kept list
    int32_t* krow = kept_idx + ((size_t)bh * C + a0 + r) * k;
    uint32_t* brow = kept_bits + ((size_t)bh * C + a0 + r) * W;
    if (kept_count && lane == 0) kept_count[(size_t)bh * C + a0 + r] = k;
    int base = 0, eqseen = 0;
    for (int i = 0; i < W; ++i) {
      const int b = i * 32 + lane;
      bool take = false, eq = false;
      if (b < Ck) {
        const uint64_t key = ordered_key(row[b]);
        const uint64_t top = L == 0 ? 0ull : (L == 64 ? key : key >> (64 - L));
        take = top > P;
        eq = top == P;
      }
      const unsigned eqb = __ballot_sync(0xffffffffu, eq);
      if (eq) take = all || (eqseen + __popc(eqb & lt) < krem);
      eqseen += __popc(eqb);
      const unsigned tb = __ballot_sync(0xffffffffu, take);
      if (lane == 0) brow[i] = tb;
      if (take) krow[base + __popc(tb & lt)] = b;
      base += __popc(tb);
    }
  }
}

template <int D, int QA>
size_t route_smem(int Ck) {
  return (size_t)QA * D * 8 + (size_t)QA * Ck * 8;
}

template <int D, int QA>
cudaError_t launch_qa(const ca_shape* s, int C, int Ck, const double* qbar, const double* kbar, int k,
                      int32_t* kept_idx, uint32_t* kept_bits, int32_t* kept_count, cudaStream_t st) {
  const size_t smem = route_smem<D, QA>(Ck);
  cudaError_t e = cudaFuncSetAttribute(route_kernel<D, QA>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((C + QA - 1) / QA, s->B * s->H);
  route_kernel<D, QA><<<grid, kRouteThreads, smem, st>>>(qbar, kbar, C, Ck, k, kept_idx, kept_bits, kept_count);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const ca_shape* s, int C, int Ck, const double* qbar, const double* kbar, int k,
                     int32_t* kept_idx, uint32_t* kept_bits, int32_t* kept_count, cudaStream_t st) {
  // as many query clusters per block as the score rows allow in the budget
  if (route_smem<D, 16>(Ck) <= kRouteSmemBudget)
    return launch_qa<D, 16>(s, C, Ck, qbar, kbar, k, kept_idx, kept_bits, kept_count, st);
  if (route_smem<D, 8>(Ck) <= kRouteSmemBudget)
    return launch_qa<D, 8>(s, C, Ck, qbar, kbar, k, kept_idx, kept_bits, kept_count, st);
  if (route_smem<D, 4>(Ck) <= kRouteSmemBudget)
    return launch_qa<D, 4>(s, C, Ck, qbar, kbar, k, kept_idx, kept_bits, kept_count, st);
  if (route_smem<D, 2>(Ck) <= kRouteSmemBudget)
    return launch_qa<D, 2>(s, C, Ck, qbar, kbar, k, kept_idx, kept_bits, kept_count, st);
  return launch_qa<D, 1>(s, C, Ck, qbar, kbar, k, kept_idx, kept_bits, kept_count, st);
}

}  // namespace

size_t route_smem_bytes(int Ck, int D) {
  return D == 64 ? route_smem<64, 1>(Ck) : route_smem<128, 1>(Ck);
}

cudaError_t launch_route(const ca_shape* s, int C, int Ck, const double* qbar, const double* kbar, int k,
                         int32_t* kept_idx, uint32_t* kept_bits, int32_t* kept_count, cudaStream_t st) {
  if (s->d == 64) return launch_d<64>(s, C, Ck, qbar, kbar, k, kept_idx, kept_bits, kept_count, st);
  return launch_d<128>(s, C, Ck, qbar, kbar, k, kept_idx, kept_bits, kept_count, st);
}

// ---------------------------------------------------------------------------
// Adaptive selection (Section 3.3.2, second method): one block per query
// cluster (C below is the number of key clusters). w_b = s_ab / sqrt(d) + ln|b| is the log of the estimated attention
// mass |b| e^{s_ab / sqrt(d)}; the key clusters are sorted by decreasing w
// (ties to the lower index, bitonic network in shared memory), their masses
// e^{w - w_max} summed in that order by one thread, and the shortest prefix
// whose running sum reaches recall x total is kept (at least min(min_count,
// C) clusters, at most the row capacity k).
// ---------------------------------------------------------------------------
namespace {

constexpr int kAdaptThreads = 256;

// bitonic width: the power of two >= C, at least 64
int adaptive_cpad(int C) {
  int p = 64;
  while (p < C) p <<= 1;
  return p;
}

template <int D>
__global__ void __launch_bounds__(kAdaptThreads) route_adaptive_kernel(
    const double* __restrict__ qbar, const double* __restrict__ kbar, const int32_t* __restrict__ count_k, int Cq,
    int C, int Cpad, double recall, int min_count, int k, int32_t* __restrict__ kept_idx,
    uint32_t* __restrict__ kept_bits, int32_t* __restrict__ kept_count) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* w = reinterpret_cast<double*>(smem_raw);             // Cpad: log masses, then masses
  int* id = reinterpret_cast<int*>(w + Cpad);                  // Cpad
  uint32_t* bits = reinterpret_cast<uint32_t*>(id + Cpad);     // Cpad / 32
  __shared__ double qa[D];
  __shared__ int kcount;
  const int a = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const double* kb = kbar + (size_t)bh * C * D;
  for (int e = t; e < D; e += kAdaptThreads) qa[e] = qbar[((size_t)bh * Cq + a) * D + e];
  for (int e = t; e < Cpad / 32; e += kAdaptThreads) bits[e] = 0u;
  __syncthreads();
  const double scale = 1.0 / sqrt((double)D);
  for (int b = t; b < Cpad; b += kAdaptThreads) {
    double v = -INFINITY;
    if (b < C) {
      const double2* kr = reinterpret_cast<const double2*>(kb + (size_t)b * D);
      double s0 = 0.0, s1 = 0.0;
#pragma unroll 8
      for (int j = 0; j < D / 2; ++j) {
        const double2 k2 = __ldg(kr + j);
        s0 = fma(qa[2 * j], k2.x, s0);
        s1 = fma(qa[2 * j + 1], k2.y, s1);
      }
      v = (s0 + s1) * scale + log((double)count_k[(size_t)bh * C + b]);
    }
    w[b] = v;
    id[b] = b < C ? b : 0x7fffffff;
  }
  __syncthreads();
  // bitonic sort: decreasing w, increasing index
  for (int size = 2; size <= Cpad; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = t; i < Cpad; i += kAdaptThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const double wi = w[i], wj = w[j];
          const int ii = id[i], ij = id[j];
          const bool i_first = (wi > wj) || (wi == wj && ii < ij);
          const bool up = ((i & size) == 0);
          if (up ? !i_first : i_first) { w[i] = wj; w[j] = wi; id[i] = ij; id[j] = ii; }
        }
      }
      __syncthreads();
    }
  }
  const double wmax = w[0];
  __syncthreads();
  for (int i = t; i < C; i += kAdaptThreads) w[i] = exp(w[i] - wmax);
  __syncthreads();
  if (t == 0) {
    double total = 0.0;
    for (int i = 0; i < C; ++i) total += w[i];
    int kk = 1;
    if (recall > 0.0) {
      const double need = recall * total;
      double cum = 0.0;
      kk = C;
      for (int i = 0; i < C; ++i) {
        cum += w[i];
        if (cum >= need) { kk = i + 1; break; }
      }
    }
    kk = max(kk, min(min_count, C));
    kcount = min(kk, k);
  }
  __syncthreads();
  const int kk = kcount;
  for (int i = t; i < kk; i += kAdaptThreads) atomicOr(&bits[id[i] >> 5], 1u << (id[i] & 31));
  __syncthreads();
  const int W = (C + 31) / 32;
  for (int e = t; e < W; e += kAdaptThreads) kept_bits[((size_t)bh * Cq + a) * W + e] = bits[e];
  if (t == 0) kept_count[(size_t)bh * Cq + a] = kk;
  // ascending kept list: one warp scans the words' popcounts, 32 at a time
  if (t < 32) {
    int32_t* krow = kept_idx + ((size_t)bh * Cq + a) * k;
    int base = 0;
    for (int w0 = 0; w0 < W; w0 += 32) {
      const int e = w0 + t;
      const uint32_t m = e < W ? bits[e] : 0u;
      const int cnt = __popc(m);
      int inc = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, inc, o);
        if (t >= o) inc += v;
      }
      int o = base + inc - cnt;
      uint32_t mm = m;
      while (mm) {
        krow[o++] = e * 32 + (__ffs(mm) - 1);
        mm &= mm - 1;
      }
      base += __shfl_sync(0xffffffffu, inc, 31);
    }
  }
}

}  // namespace

size_t route_adaptive_smem(int Ck) {
  const int Cpad = adaptive_cpad(Ck);
  return (size_t)Cpad * 12 + (size_t)(Cpad / 32) * 4;
}

// Cq query clusters (one block each), C key clusters.
cudaError_t launch_route_adaptive(const ca_shape* s, int Cq, int C, const double* qbar, const double* kbar,
                                  const int32_t* count_k, double recall, int min_count, int k, int32_t* kept_idx,
                                  uint32_t* kept_bits, int32_t* kept_count, cudaStream_t st) {
  const int Cpad = adaptive_cpad(C);
  const size_t smem = route_adaptive_smem(C);
  const dim3 grid(Cq, s->B * s->H);
  cudaError_t e;
  if (s->d == 64) {
    e = cudaFuncSetAttribute(route_adaptive_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    route_adaptive_kernel<64><<<grid, kAdaptThreads, smem, st>>>(qbar, kbar, count_k, Cq, C, Cpad, recall, min_count, k,
                                                                 kept_idx, kept_bits, kept_count);
  } else {
    e = cudaFuncSetAttribute(route_adaptive_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    route_adaptive_kernel<128><<<grid, kAdaptThreads, smem, st>>>(qbar, kbar, count_k, Cq, C, Cpad, recall, min_count,
                                                                  k, kept_idx, kept_bits, kept_count);
  }
  return cudaGetLastError();
}

}  // namespace ca
