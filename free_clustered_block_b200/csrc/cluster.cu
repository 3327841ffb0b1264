// Clustering kernels: metric matrices, per-node principal direction by power
// iteration, projection, radix select of the split threshold, stable
// partition, centroids.
//
// ClusterAttention paper, Section 3.2 "Clustering" (3.2.1 basic recursive
// splitting, 3.2.2 transforms) and Section 6.1 (the metric matrix injected
// into the power iteration instead of an eigendecomposition).
//
// Arithmetic that decides the partition is fp64 throughout: inputs (bf16 or
// fp32) widen exactly to fp64, metric matrices, query norms, directions and
// projections are fp64, and the split is an exact order statistic of the
// fp64 projections, equal values ordered by row index.
#include "ca_internal.cuh"

namespace ca {

namespace {

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// Tensor-head of a block: th = 2 bh + tensor. With tsel < 0 the grid row y
// enumerates every tensor-head (both tensors, one tree); with tsel = 0 or 1
// it enumerates the heads of that tensor alone (each tensor walks its own
// tree when the query and key cluster sizes differ).
__device__ __forceinline__ int tensor_head(int y, int tsel) { return tsel < 0 ? y : 2 * y + tsel; }

// Warp sum of a double, fixed butterfly order (deterministic).
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// Tree tables on the device: breadth first, one level at a time; the
// children of node i land at (level end + exclusive prefix of the child
// counts), which reproduces the host's sequential plan_tree order exactly.
// One block of 1024 threads.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) plan_kernel(int n, int c, TreeNode* nodes, int* level_begin) {
  __shared__ int warp_tot[32];
  __shared__ int s_total;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (n <= c) {
    if (tid == 0) level_begin[0] = 0;
    return;
  }
  if (tid == 0) {
    TreeNode r;
    r.off = 0; r.size = n; r.t = split_count(n, c); r.parent = -1; r.heap = 1;
    nodes[0] = r;
  }
  __syncthreads();
  int begin = 0, end = 1, count = 1, lvl = 0;
  while (begin < end && lvl < kMaxLevels) {
    if (tid == 0) level_begin[lvl] = begin;
    for (int chunk = begin; chunk < end; chunk += 1024) {
      const int i = chunk + tid;
      TreeNode nd;
      int ls = 0, rs = 0, nch = 0;
      if (i < end) {
        nd = nodes[i];
        ls = nd.t; rs = nd.size - nd.t;
        nch = (ls > c) + (rs > c);
      }
      int x = nch;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) warp_tot[warp] = x;
      __syncthreads();
      if (warp == 0) {
        int t = warp_tot[lane];
        int u = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, u, o);
          if (lane >= o) u += y;
        }
        warp_tot[lane] = u - t;
        if (lane == 31) s_total = u;
      }
      __syncthreads();
      if (i < end) {
        int pos = count + warp_tot[warp] + x - nch;
        if (ls > c) {
          TreeNode ch;
          ch.off = nd.off; ch.size = ls; ch.t = split_count(ls, c); ch.parent = i; ch.heap = 2 * nd.heap;
          nodes[pos++] = ch;
        }
        if (rs > c) {
          TreeNode ch;
          ch.off = nd.off + ls; ch.size = rs; ch.t = split_count(rs, c); ch.parent = i; ch.heap = 2 * nd.heap + 1;
          nodes[pos] = ch;
        }
      }
      count += s_total;
      __syncthreads();
    }
    begin = end; end = count; ++lvl;
  }
  if (tid == 0) level_begin[lvl] = count;
}

// ---------------------------------------------------------------------------
// S1: column sums of K (for the key mean), per row chunk.
// ---------------------------------------------------------------------------
// With kW the rows are scaled by w[bh n + row] first (the queries' 1 / |R_k q|
// for the covariance of their representations).
template <typename T, int D, bool kW = false>
__global__ void __launch_bounds__(256) colsum_kernel(const T* __restrict__ K, TensorLayout TL, int n,
                                                     double* __restrict__ part,
                                                     const double* __restrict__ w = nullptr) {
  constexpr int RG = 256 / D;
  const int bh = blockIdx.y, ch = blockIdx.x, nch = gridDim.x;
  const int r0 = ch * kMetricChunk, r1 = min(n, r0 + kMetricChunk);
  const int col = threadIdx.x % D, rg = threadIdx.x / D;
  const T* base = K + TL.head(bh);
  double acc = 0.0;
  // rows r0 + rg, r0 + rg + RG, ... summed in that order, four loads in flight
  const size_t step = (size_t)RG * TL.sn;
  const T* src = base + (size_t)(r0 + rg) * TL.sn + col;
  int r = r0 + rg;
  for (; r + 3 * RG < r1; r += 4 * RG, src += 4 * step) {
    const T x0 = src[0], x1 = src[step], x2 = src[2 * step], x3 = src[3 * step];
    if constexpr (kW) {
      const double* wr = w + (size_t)bh * n + r;
      acc = fma((double)to_f(x0), wr[0], acc);
      acc = fma((double)to_f(x1), wr[RG], acc);
      acc = fma((double)to_f(x2), wr[2 * RG], acc);
      acc = fma((double)to_f(x3), wr[3 * RG], acc);
    } else {
      acc += (double)to_f(x0);
      acc += (double)to_f(x1);
      acc += (double)to_f(x2);
      acc += (double)to_f(x3);
    }
  }
  for (; r < r1; r += RG, src += step) {
    if constexpr (kW) acc = fma((double)to_f(src[0]), w[(size_t)bh * n + r], acc);
    else acc += (double)to_f(src[0]);
  }
  __shared__ double red[256];
  red[threadIdx.x] = acc;
  __syncthreads();
  if (rg == 0) {
    double s = 0.0;
    for (int g = 0; g < RG; ++g) s += red[g * D + col];
    part[((size_t)bh * nch + ch) * D + col] = s;
  }
}

// ---------------------------------------------------------------------------
// S1: partial second-moment matrices over a row chunk, on the fp64 CUDA
// cores (the weighted query covariance of the diagonalized splitting; the
// metrics themselves use syrk_mma_kernel below).
// z = 0: Q^T Q (uncentred); z = 1: (K - kmean)^T (K - kmean).
// Only the upper triangle of 8 x 8 tiles is accumulated (the matrix is
// symmetric): thread t of row group g owns tile t over the staged rows
// g, g + R, g + 2R, ... The R groups are then summed in a fixed order through
// shared memory, so the result does not depend on scheduling.
// Rows arrive by 16-byte cp.async into a raw tile while the previous tile is
// being multiplied, and are converted (minus the mean) into an fp64 tile whose
// 16-byte chunks are rotated within each 8-column group, so that the lanes of
// a warp reading chunk i of different column groups hit different banks.
// ---------------------------------------------------------------------------
template <int D>
struct SyrkCfg {
  static constexpr int TR = D / 8;                 // 8-row tile rows
  static constexpr int TC = D / 4;                 // 4-column tile columns
  static constexpr int NT = TR * TC - TR * (TR - 1);   // tiles (I, J) with 4J + 3 >= 8I: 72 / 272
  static constexpr int R = D == 64 ? 3 : 1;        // row groups
  static constexpr int kThreads = NT * R;          // 216 (d = 64), 272 (d = 128)
  static constexpr int kRows = D == 64 ? 63 : 32;  // rows staged per step (a multiple of R)
  static constexpr size_t kXsBytes = (size_t)kRows * D * 8 > (R > 1 ? (size_t)D * D * 8 : 0)
                                         ? (size_t)kRows * D * 8
                                         : (size_t)D * D * 8;
  template <typename T>
  static constexpr size_t smem() { return kXsBytes + (size_t)kRows * D * sizeof(T); }
};

// position (in doubles) of column col inside a staged fp64 row
__device__ __forceinline__ int syrk_pos(int col) {
  const int I = col >> 3, i = (col >> 1) & 3;
  return ((4 * I + ((i + (I >> 1)) & 3)) << 1) | (col & 1);
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// kW: one launch over the queries only (grid.z = 1), rows scaled by
// w[bh n + row] and centred by the weighted mean taken from colpart; the
// result goes to the queries' slot (z = 0) of part. This is the covariance of
// the query representations before the transform (diagonalized splitting).
template <typename T, int D, bool kW = false>
__global__ void __maxnreg__(128) syrk_kernel(const T* __restrict__ Q, const T* __restrict__ K, TensorLayout TL,
                                             int n, int nch, const double* __restrict__ colpart,
                                             double* __restrict__ part, const double* __restrict__ w = nullptr) {
  using Cfg = SyrkCfg<D>;
  constexpr int R = Cfg::R, NTH = Cfg::kThreads, ROWS = Cfg::kRows;
  constexpr int VEC = 16 / sizeof(T);                 // elements per 16-byte chunk
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* xs = reinterpret_cast<double*>(smem_raw);   // ROWS x D (rotated), later D x D for the group sum
  T* raw = reinterpret_cast<T*>(smem_raw + Cfg::kXsBytes);   // ROWS x D as loaded
  __shared__ double mean[D];
  const int bh = blockIdx.y, z = blockIdx.z, ch = blockIdx.x;
  const T* X = (z == 0 ? Q : K) + TL.head(bh);
  const int r0 = ch * kMetricChunk, r1 = min(n, r0 + kMetricChunk);

  auto issue = [&](int rt) {
    const int rows = min(ROWS, r1 - rt);
    for (int e = threadIdx.x; e < rows * (D / VEC); e += NTH)
      cp_async16(raw + e * VEC, X + (size_t)(rt + e / (D / VEC)) * TL.sn + (size_t)(e % (D / VEC)) * VEC);
    cp_async_commit();
  };
  if (r0 < r1) issue(r0);
  for (int c = threadIdx.x; c < D; c += NTH) {
    double m = 0.0;
    if (kW || z == 1) {
      for (int i = 0; i < nch; ++i) m += colpart[((size_t)bh * nch + i) * D + c];
      m /= (double)n;
    }
    mean[c] = m;
  }
  // tile t -> (I, J): rows 8I..8I+7, columns 4J..4J+3, J >= 2I (on or above the diagonal)
  const int g = threadIdx.x / Cfg::NT, t = threadIdx.x % Cfg::NT;
  int I = 0, rem = t;
  while (rem >= Cfg::TC - 2 * I) { rem -= Cfg::TC - 2 * I; ++I; }
  const int J = 2 * I + rem;
  const int JI = J >> 1, Jc = 2 * (J & 1);             // 8-column group and first chunk of it
  double acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
  for (int rt = r0; rt < r1; rt += ROWS) {
    cp_async_wait_all();
    __syncthreads();   // raw tile complete, mean written, previous tile's products done
    const int rows = min(ROWS, r1 - rt);
    for (int e = threadIdx.x; e < ROWS * D; e += NTH) {
      const int rr = e / D, cc = e % D;
      if constexpr (kW)
        xs[rr * D + syrk_pos(cc)] =
            rr < rows ? (double)to_f(raw[e]) * w[(size_t)bh * n + rt + rr] - mean[cc] : 0.0;
      else
        xs[rr * D + syrk_pos(cc)] = rr < rows ? (double)to_f(raw[e]) - mean[cc] : 0.0;
    }
    __syncthreads();
    if (rt + ROWS < r1) issue(rt + ROWS);
#pragma unroll (D == 64 ? 2 : 1)
    for (int rr = g; rr < ROWS; rr += R) {
      const double2* row = reinterpret_cast<const double2*>(xs + rr * D);
      double a[8], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const double2 va = row[4 * I + ((i + (I >> 1)) & 3)];
        a[2 * i] = va.x; a[2 * i + 1] = va.y;
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const double2 vb = row[4 * JI + ((Jc + i + (JI >> 1)) & 3)];
        b[2 * i] = vb.x; b[2 * i + 1] = vb.y;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
  }
  double* out = part + (((size_t)bh * 2 + z) * nch + ch) * D * D;
  // an entry (r, c) with c >= r lies in exactly one tile; write it and its mirror
  if constexpr (R == 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = 8 * I + i, c = 4 * J + j;
        if (c >= r) { out[r * D + c] = acc[i][j]; out[c * D + r] = acc[i][j]; }
      }
  } else {
    __syncthreads();    // last tile's products done before xs becomes the group sum
    double* red = xs;   // D x D, entries (r, c >= r)
    for (int gg = 0; gg < R; ++gg) {
      if (g == gg) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int r = 8 * I + i, c = 4 * J + j;
            if (c >= r) red[r * D + c] = (gg == 0 ? 0.0 : red[r * D + c]) + acc[i][j];
          }
      }
      __syncthreads();
    }
    for (int e = threadIdx.x; e < D * D; e += NTH) {
      const int i = e / D, j = e % D;
      out[e] = j >= i ? red[e] : red[j * D + i];
    }
  }
}

// The same partial second-moment matrices on the fp64 tensor-core path
// (mma.sync m8n8k4 f64): the upper triangle of 32 x 32 blocks, one warp per
// (block, row group); per step of four rows a warp loads four A and four B
// fragments (one double per lane each) and issues sixteen 8 x 8 x 4 products,
// so shared memory delivers half a byte per FMA instead of three for the
// 8 x 4 register tiles of syrk_kernel. Rows are staged as in syrk_kernel
// (cp.async of the raw rows while the previous tile is multiplied, then one
// conversion to fp64 minus the mean); the row groups are summed in a fixed
// order through shared memory.
template <int D>
struct SyrkMmaCfg {
  static constexpr int NB = D / 32;                   // 32-wide blocks per dimension
  static constexpr int NBT = NB * (NB + 1) / 2;       // blocks on or above the diagonal: 3 / 10
  static constexpr int RG = D == 64 ? 4 : 1;          // row groups
  static constexpr int kWarps = NBT * RG;             // 12 / 10
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kRows = 64;                    // rows staged per step (a multiple of 4 RG)
  static constexpr int kP = D + 4;                    // fp64 row stride: fragment loads hit distinct banks
  static constexpr size_t kXsBytes = (size_t)kRows * kP * 8 > (RG > 1 ? (size_t)D * D * 8 : 0)
                                         ? (size_t)kRows * kP * 8
                                         : (size_t)D * D * 8;
  template <typename T>
  static constexpr size_t smem() { return kXsBytes + (size_t)kRows * D * sizeof(T); }
};

__device__ __forceinline__ void dmma_884(double (&c)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(c[0]), "+d"(c[1])
               : "d"(a), "d"(b));
}

template <typename T, int D>
__global__ void __launch_bounds__(SyrkMmaCfg<D>::kThreads, 1) syrk_mma_kernel(
    const T* __restrict__ Q, const T* __restrict__ K, TensorLayout TL, int n, int nch,
    const double* __restrict__ colpart, double* __restrict__ part) {
  using Cfg = SyrkMmaCfg<D>;
  constexpr int RG = Cfg::RG, NTH = Cfg::kThreads, ROWS = Cfg::kRows, P = Cfg::kP;
  constexpr int VEC = 16 / sizeof(T);
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* xs = reinterpret_cast<double*>(smem_raw);            // ROWS x P, later D x D for the group sum
  T* raw = reinterpret_cast<T*>(smem_raw + Cfg::kXsBytes);     // ROWS x D as loaded
  __shared__ double mean[D];
  const int bh = blockIdx.y, z = blockIdx.z, ch = blockIdx.x;
  const T* X = (z == 0 ? Q : K) + TL.head(bh);
  const int r0 = ch * kMetricChunk, r1 = min(n, r0 + kMetricChunk);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, tg = lane & 3;                      // fragment row / column in group
  const int rg = warp / Cfg::NBT, blk = warp % Cfg::NBT;
  int bi = 0, rem = blk;                                       // block (bi, bj), bj >= bi
  while (rem >= Cfg::NB - bi) { rem -= Cfg::NB - bi; ++bi; }
  const int bj = bi + rem;

  auto issue = [&](int rt) {
    const int rows = min(ROWS, r1 - rt);
    for (int e = threadIdx.x; e < rows * (D / VEC); e += NTH)
      cp_async16(raw + e * VEC, X + (size_t)(rt + e / (D / VEC)) * TL.sn + (size_t)(e % (D / VEC)) * VEC);
    cp_async_commit();
  };
  if (r0 < r1) issue(r0);
  for (int c = threadIdx.x; c < D; c += NTH) {
    double m = 0.0;
    if (z == 1) {
      for (int i = 0; i < nch; ++i) m += colpart[((size_t)bh * nch + i) * D + c];
      m /= (double)n;
    }
    mean[c] = m;
  }
  double acc[4][4][2];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b][0] = acc[a][b][1] = 0.0;
  for (int rt = r0; rt < r1; rt += ROWS) {
    cp_async_wait_all();
    __syncthreads();   // raw tile complete, mean written, previous tile's products done
    const int rows = min(ROWS, r1 - rt);
    for (int e = threadIdx.x; e < ROWS * D; e += NTH) {
      const int rr = e / D, cc = e % D;
      xs[rr * P + cc] = rr < rows ? (double)to_f(raw[e]) - mean[cc] : 0.0;
    }
    __syncthreads();
    if (rt + ROWS < r1) issue(rt + ROWS);
#pragma unroll 2
    for (int k0 = 4 * rg; k0 < ROWS; k0 += 4 * RG) {
      const double* xr = xs + (k0 + tg) * P;
      double fa[4], fb[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) fa[a] = xr[32 * bi + 8 * a + g];
#pragma unroll
      for (int b = 0; b < 4; ++b) fb[b] = xr[32 * bj + 8 * b + g];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) dmma_884(acc[a][b], fa[a], fb[b]);
    }
  }
  double* out = part + (((size_t)bh * 2 + z) * nch + ch) * D * D;
  // this lane's entries: row 32 bi + 8 a + g, columns 32 bj + 8 b + 2 tg + {0, 1}
  if constexpr (RG == 1) {
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int r = 32 * bi + 8 * a + g, c = 32 * bj + 8 * b + 2 * tg + i;
          if (c >= r) { out[r * D + c] = acc[a][b][i]; out[c * D + r] = acc[a][b][i]; }
        }
  } else {
    __syncthreads();    // last tile's products done before xs becomes the group sum
    double* red = xs;   // D x D, entries (r, c >= r)
    for (int gg = 0; gg < RG; ++gg) {
      if (rg == gg) {
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int r = 32 * bi + 8 * a + g, c = 32 * bj + 8 * b + 2 * tg + i;
              if (c >= r) red[r * D + c] = (gg == 0 ? 0.0 : red[r * D + c]) + acc[a][b][i];
            }
      }
      __syncthreads();
    }
    for (int e = threadIdx.x; e < D * D; e += NTH) {
      const int i = e / D, j = e % D;
      out[e] = j >= i ? red[e] : red[j * D + i];
    }
  }
}

// M[th] for tensor-head th = 2 bh + tensor: queries (tensor 0) are split in
// the key metric M_k, keys (tensor 1) in the query metric M_q. One thread
// per matrix element (grid.x covers D*D / 256), the chunk partials summed in
// chunk order with four loads in flight.
template <int D>
__global__ void __launch_bounds__(256) metric_reduce_kernel(const double* __restrict__ part, int nch,
                                                            int n, int transform,
                                                            double* __restrict__ M) {
  const int th = blockIdx.y, bh = th >> 1, tensor = th & 1;
  const int src = 1 - tensor;  // z index: 0 = Q^T Q, 1 = K_c^T K_c
  const double* p = part + ((size_t)bh * 2 + src) * nch * D * D;
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e >= D * D) return;
  double v;
  if (transform) {
    v = 0.0;
    int ch = 0;
    for (; ch + 4 <= nch; ch += 4) {
      const double a0 = p[(size_t)ch * D * D + e], a1 = p[(size_t)(ch + 1) * D * D + e];
      const double a2 = p[(size_t)(ch + 2) * D * D + e], a3 = p[(size_t)(ch + 3) * D * D + e];
      v += a0; v += a1; v += a2; v += a3;
    }
    for (; ch < nch; ++ch) v += p[(size_t)ch * D * D + e];
    v /= (double)n;
  } else {
    v = (e / D == e % D) ? 1.0 : 0.0;
  }
  M[(size_t)th * D * D + e] = v;
}

// ---------------------------------------------------------------------------
// Query scale 1/|R_k q| = 1/sqrt(q^T M_k q) (eq. 16), 0 when q^T M_k q <= 0.
// 128 rows per block; thread (ty,tx) computes T = X M for rows ty+16i, cols
// tx+16j, then the row dot with X.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256) qnorm_kernel(const T* __restrict__ Q, TensorLayout TL, int n,
                                                    const double* __restrict__ M, int transform,
                                                    double* __restrict__ inv_s) {
  constexpr int R = 128, B = D / 16, RS = D + 1;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* Ms = reinterpret_cast<double*>(smem_raw);           // [D][D]
  float* xs = reinterpret_cast<float*>(Ms + D * D);           // [R][D+1]
  const int bh = blockIdx.y, r0 = blockIdx.x * R;
  const int th = bh * 2;  // queries use M_k, stored at the queries' tensor-head
  if (!transform) {
    for (int r = threadIdx.x; r < R; r += 256)
      if (r0 + r < n) inv_s[(size_t)bh * n + r0 + r] = 1.0;
    return;
  }
  for (int e = threadIdx.x; e < D * D; e += 256) Ms[e] = M[(size_t)th * D * D + e];
  const T* X = Q + TL.head(bh);
  for (int e = threadIdx.x; e < R * D; e += 256) {
    const int rr = e / D, cc = e % D, r = r0 + rr;
    xs[rr * RS + cc] = (r < n) ? to_f(X[(size_t)r * TL.sn + cc]) : 0.f;
  }
  __syncthreads();
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  constexpr int RI = R / 16;  // 8 rows per thread
  double acc[RI][B];
#pragma unroll
  for (int i = 0; i < RI; ++i)
#pragma unroll
    for (int j = 0; j < B; ++j) acc[i][j] = 0.0;
#pragma unroll 2
  for (int k = 0; k < D; ++k) {
    double a[RI], b[B];
#pragma unroll
    for (int i = 0; i < RI; ++i) a[i] = (double)xs[(ty + 16 * i) * RS + k];
#pragma unroll
    for (int j = 0; j < B; ++j) b[j] = Ms[k * D + tx + 16 * j];
#pragma unroll
    for (int i = 0; i < RI; ++i)
#pragma unroll
      for (int j = 0; j < B; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < RI; ++i) {
    double s = 0.0;
#pragma unroll
    for (int j = 0; j < B; ++j) s = fma(acc[i][j], (double)xs[(ty + 16 * i) * RS + tx + 16 * j], s);
    // reduce over the 16 lanes sharing ty (lanes 0-15 / 16-31 of the warp)
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const int r = r0 + ty + 16 * i;
    if (tx == 0 && r < n) inv_s[(size_t)bh * n + r] = (s > 0.0) ? 1.0 / sqrt(s) : 0.0;
  }
}

// d = 64 variant: one thread per query row, the row held in registers as
// fp64. q^T M q = sum_i q_i (M_ii q_i + 2 sum_{j>i} M_ij q_j) uses only the
// upper triangle of the symmetric M (2080 fma per row instead of 4160); every
// lane reads the same M entries, so the shared-memory loads are broadcasts.
template <typename T>
__global__ void __launch_bounds__(128, 3) qnorm64_kernel(const T* __restrict__ Q, TensorLayout TL, int n,
                                                      const double* __restrict__ M,
                                                      double* __restrict__ inv_s) {
  constexpr int D = 64;
  __shared__ __align__(16) double Ms[D * D];
  const int bh = blockIdx.y, r = blockIdx.x * 128 + threadIdx.x;
  const double* Mh = M + (size_t)(bh * 2) * D * D;   // queries use M_k
  for (int e = threadIdx.x; e < D * D / 2; e += 128)
    reinterpret_cast<double2*>(Ms)[e] = reinterpret_cast<const double2*>(Mh)[e];
  double x[D];
  {
    constexpr int VEC = 16 / sizeof(T);
    const uint4* src = reinterpret_cast<const uint4*>(Q + TL.head(bh) + (size_t)(r < n ? r : 0) * TL.sn);
    uint4 raw[D / VEC];
#pragma unroll
    for (int v = 0; v < D / VEC; ++v) raw[v] = __ldg(src + v);
#pragma unroll
    for (int v = 0; v < D / VEC; ++v) {
      const T* e = reinterpret_cast<const T*>(&raw[v]);
#pragma unroll
      for (int u = 0; u < VEC; ++u) x[v * VEC + u] = (double)to_f(e[u]);
    }
  }
  __syncthreads();
  if (r >= n) return;
  double s = 0.0;
#pragma unroll
  for (int i = 0; i < D; ++i) {
    const double* Mi = Ms + i * D;
    double t0 = 0.0, t1 = 0.0;
    int j = i + 1;
    if (j & 1) { t0 = Mi[j] * x[j]; ++j; }
#pragma unroll
    for (; j < D; j += 2) {
      const double2 m2 = *reinterpret_cast<const double2*>(Mi + j);
      t0 = fma(m2.x, x[j], t0);
      t1 = fma(m2.y, x[j + 1], t1);
    }
    s = fma(x[i], fma(2.0, t0 + t1, Mi[i] * x[i]), s);
  }
  inv_s[(size_t)bh * n + r] = (s > 0.0) ? 1.0 / sqrt(s) : 0.0;
}

// ---------------------------------------------------------------------------
// K1: per-node principal direction by power iteration, metric injected.
//
// With the transformed vectors y = R x (R = sqrt(M)), the sample covariance
// is C_y = R C_x R. Writing the iterate as u = R z, u <- C_y u becomes
// z <- C_x M z and |u|^2 = z^T M z; the projection y . u = x^T (M z). So the
// node's direction for projection is w = M z, with no root or eigenproblem.
// Queries use x = q / |R_k q| (eq. 16).
// Warm start (Section 3.2.1): mean of the parent's (unit) estimate and a
// random normal vector of unit norm; g is drawn in the untransformed
// coordinates and mapped through R: g_hat = R g / |R g|, i.e. z_g = g / sqrt(g^T M g).
// ---------------------------------------------------------------------------
// One warp per node: the block's warps take consecutive nodes of one
// tensor-head and share its M in shared memory; each warp stages its node's
// sample rows (in the input type, exact) in shared memory with a padded row
// stride (odd number of 32-bit words, conflict-free both along rows and
// along columns). Every reduction is a warp shuffle: after M is staged no
// block barrier is needed.
template <typename T, int D>
struct DirCfg {
  static constexpr int kRowPad = (sizeof(T) == 2) ? 2 : 1;             // elements
  static constexpr int kRowStride = D + kRowPad;                       // elements; odd word count
  __host__ __device__ static size_t warp_bytes(int m_cap) {
    return (size_t)m_cap * kRowStride * sizeof(T) + (size_t)(2 * D + 2 * m_cap) * 8 + (size_t)m_cap * 4;
  }
  static int warps(int m_cap) {
    const long long per = (long long)warp_bytes(m_cap);
    const long long two = 112 * 1024 - (long long)D * D * 8;   // two blocks per SM when it fits
    long long w = two > 0 ? two / per : 0;
    if (w < 1) w = (220 * 1024 - (long long)D * D * 8) / per;  // one block per SM
    if (w < 1) w = 1;
    return (int)(w > 16 ? 16 : w);
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(512) dir_kernel(
    const T* __restrict__ Q, const T* __restrict__ K, TensorLayout TL, int n, const TreeNode* __restrict__ nodes,
    int lvl_begin, int nodes_in_level, const double* __restrict__ M, const double* __restrict__ inv_s,
    const int* __restrict__ idx, int NI, double* __restrict__ zvec, double* __restrict__ wvec, uint64_t seed,
    int head_base, int power_iters, int sample_factor, int tsel) {
  using Cfg = DirCfg<T, D>;
  constexpr int CPL = D / 32;                      // coordinates per lane: a = lane + 32 c
  constexpr int RS = Cfg::kRowStride;
  const int m_cap = sample_factor * D;
  const int nwarps = blockDim.x >> 5;
  const int th = tensor_head(blockIdx.y, tsel), bh = th >> 1, tensor = th & 1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* Ms = reinterpret_cast<double*>(smem_raw);                          // D*D
  unsigned char* wbase = smem_raw + (size_t)D * D * 8 + (size_t)warp * Cfg::warp_bytes(m_cap);
  double* vz = reinterpret_cast<double*>(wbase);   // z (D)
  double* vw = vz + D;                             // w (D)
  double* vv = vw + D;                             // v over the sample (m_cap)
  double* vs = vv + m_cap;                         // sample scales (m_cap)
  int* srow = reinterpret_cast<int*>(vs + m_cap);  // sample rows (m_cap)
  T* Xs = reinterpret_cast<T*>(srow + m_cap);      // m_cap x RS sample (4-byte aligned)
  for (int e = threadIdx.x; e < D * D; e += nwarps * 32) Ms[e] = M[(size_t)th * D * D + e];
  __syncthreads();
  const int local = blockIdx.x * nwarps + warp;
  if (local >= nodes_in_level) return;             // whole warp leaves; no block barrier follows
  const int node_id = lvl_begin + local;
  const TreeNode nd = nodes[node_id];
  const int m = min(m_cap, nd.size);
  const uint64_t key = node_stream(seed, (uint64_t)(head_base + bh), (uint64_t)tensor, nd.heap);
  const uint64_t r = (nd.size > m) ? (splitmix64(key ^ kSampleTag) % (uint64_t)nd.size) : 0ull;
  const T* X = (tensor == 0 ? Q : K) + TL.head(bh);
  const int* idx_th = idx ? idx + (size_t)th * n : nullptr;
  for (int j = lane; j < m; j += 32) {
    const int pos = (nd.size > m) ? (int)(((uint64_t)j * (uint64_t)nd.size + r) / (uint64_t)m) : j;
    const int row = idx_th ? idx_th[nd.off + pos] : nd.off + pos;
    srow[j] = row;
    vs[j] = (tensor == 0) ? inv_s[(size_t)bh * n + row] : 1.0;
  }
  __syncwarp();
  // stage the sample: 16-byte chunks, several rows per warp instruction, up to
  // four instructions' loads in flight before their stores
  {
    constexpr int CPR = D * (int)sizeof(T) / 16;    // 16-byte chunks per row
    constexpr int RPI = 32 / CPR;                   // rows per warp instruction
    constexpr int WRS = RS * (int)sizeof(T) / 4;    // padded row stride in 32-bit words
    uint32_t* xw = reinterpret_cast<uint32_t*>(Xs);
    const int sub = lane / CPR, part = lane % CPR;
    for (int j0 = 0; j0 < m; j0 += 4 * RPI) {
      uint4 v4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + u * RPI + sub;
        v4[u] = make_uint4(0, 0, 0, 0);
        if (j < m) v4[u] = *reinterpret_cast<const uint4*>(X + (size_t)srow[j] * TL.sn + part * (16 / sizeof(T)));
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + u * RPI + sub;
        if (j < m) {
          uint32_t* dst = xw + (size_t)j * WRS + part * 4;
          dst[0] = v4[u].x; dst[1] = v4[u].y; dst[2] = v4[u].z; dst[3] = v4[u].w;
        }
      }
    }
  }
  __syncwarp();
  // sample mean
  double xbar[CPL];
#pragma unroll
  for (int cc = 0; cc < CPL; ++cc) xbar[cc] = 0.0;
  for (int j = 0; j < m; ++j) {
    const double sj = vs[j];
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc) xbar[cc] = fma(sj, (double)to_f(Xs[j * RS + lane + 32 * cc]), xbar[cc]);
  }
#pragma unroll
  for (int cc = 0; cc < CPL; ++cc) xbar[cc] /= (double)m;
  // w = M z with z in vz; M symmetric, column access is conflict-free
  auto matvec = [&](double* out) {
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc) {
      const int a = lane + 32 * cc;
      double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
#pragma unroll 4
      for (int b = 0; b < D; b += 4) {
        s0 = fma(Ms[b * D + a], vz[b], s0);
        s1 = fma(Ms[(b + 1) * D + a], vz[b + 1], s1);
        s2 = fma(Ms[(b + 2) * D + a], vz[b + 2], s2);
        s3 = fma(Ms[(b + 3) * D + a], vz[b + 3], s3);
      }
      out[cc] = (s0 + s1) + (s2 + s3);
    }
  };
  // z0 = (z_parent + g / sqrt(g^T M g)) / 2, or g / sqrt(g^T M g) at the root
  double g[CPL], w[CPL], z[CPL];
#pragma unroll
  for (int cc = 0; cc < CPL; ++cc) {
    const int a = lane + 32 * cc;
    // Box-Muller on two SplitMix64 draws per coordinate
    const uint64_t ua = splitmix64(key + 2ull * a + 1ull);
    const uint64_t ub = splitmix64(key + 2ull * a + 2ull);
    const double u1 = (double)((ua >> 11) + 1ull) * 0x1.0p-53;
    const double u2 = (double)(ub >> 11) * 0x1.0p-53;
    g[cc] = sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
    vz[a] = g[cc];
  }
  __syncwarp();
  matvec(w);
  double gq = 0.0;
#pragma unroll
  for (int cc = 0; cc < CPL; ++cc) gq = fma(g[cc], w[cc], gq);
  gq = warp_sum(gq);
  const double gi = (gq > 0.0) ? 1.0 / sqrt(gq) : 0.0;
#pragma unroll
  for (int cc = 0; cc < CPL; ++cc) {
    const double gh = g[cc] * gi;
    z[cc] = (nd.parent < 0) ? gh : 0.5 * (zvec[((size_t)th * NI + nd.parent) * D + lane + 32 * cc] + gh);
  }
  __syncwarp();
#pragma unroll
  for (int cc = 0; cc < CPL; ++cc) vz[lane + 32 * cc] = z[cc];
  __syncwarp();
  // power iteration in z-form: z <- C_x M z, normalised by sqrt(z^T M z)
  for (int it = 0; it < power_iters; ++it) {
    matvec(w);
    double q = 0.0, xw = 0.0;
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc) { q = fma(z[cc], w[cc], q); xw = fma(xbar[cc], w[cc], xw); }
    q = warp_sum(q);
    xw = warp_sum(xw);
    const double s = (q > 0.0) ? 1.0 / sqrt(q) : 0.0;
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc) vw[lane + 32 * cc] = w[cc];
    __syncwarp();
    // v_j = s (scale_j X_j . w - xbar . w); lane takes rows j = lane + 32 q
    double vsum = 0.0;
    for (int j = lane; j < m; j += 32) {
      const T* xr = Xs + j * RS;
      double d0 = 0.0, d1 = 0.0, d2 = 0.0, d3 = 0.0;
#pragma unroll 4
      for (int e = 0; e < D; e += 4) {
        d0 = fma((double)to_f(xr[e]), vw[e], d0);
        d1 = fma((double)to_f(xr[e + 1]), vw[e + 1], d1);
        d2 = fma((double)to_f(xr[e + 2]), vw[e + 2], d2);
        d3 = fma((double)to_f(xr[e + 3]), vw[e + 3], d3);
      }
      const double vj = s * fma(vs[j], (d0 + d1) + (d2 + d3), -xw);
      vv[j] = vj;
      vsum += vj;
    }
    vsum = warp_sum(vsum);
    __syncwarp();
    // z'_a = (sum_j v_j scale_j X_ja - xbar_a sum_j v_j) / m
    double acc0[CPL], acc1[CPL];
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc) { acc0[cc] = 0.0; acc1[cc] = 0.0; }
    int j = 0;
    for (; j + 1 < m; j += 2) {
      const double f0 = vv[j] * vs[j], f1 = vv[j + 1] * vs[j + 1];
#pragma unroll
      for (int cc = 0; cc < CPL; ++cc) {
        acc0[cc] = fma(f0, (double)to_f(Xs[j * RS + lane + 32 * cc]), acc0[cc]);
        acc1[cc] = fma(f1, (double)to_f(Xs[(j + 1) * RS + lane + 32 * cc]), acc1[cc]);
      }
    }
    if (j < m) {
      const double f0 = vv[j] * vs[j];
#pragma unroll
      for (int cc = 0; cc < CPL; ++cc) acc0[cc] = fma(f0, (double)to_f(Xs[j * RS + lane + 32 * cc]), acc0[cc]);
    }
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc) z[cc] = ((acc0[cc] + acc1[cc]) - xbar[cc] * vsum) / (double)m;
    __syncwarp();
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc) vz[lane + 32 * cc] = z[cc];
    __syncwarp();
  }
  matvec(w);
  double q = 0.0;
#pragma unroll
  for (int cc = 0; cc < CPL; ++cc) q = fma(z[cc], w[cc], q);
  q = warp_sum(q);
  const double qi = (q > 0.0) ? 1.0 / sqrt(q) : 0.0;
#pragma unroll
  for (int cc = 0; cc < CPL; ++cc) {
    const size_t o = ((size_t)th * NI + node_id) * D + lane + 32 * cc;
    zvec[o] = z[cc] * qi;
    wvec[o] = w[cc] * qi;
  }
}

// One block of 2 d threads per node (a sample of at most d rows), walking
// `npc` consecutive nodes of one tensor-head with M staged once. Used for
// d = 128, where M alone is 128 KB and one warp per node would leave two
// nodes per SM, and for d = 64 on the levels with few nodes, where one warp
// per node is latency-bound. Each of the three products of a power step is
// split over the threads as pairs of half sums (rows or columns 0..d/2-1 and
// d/2..d-1), added in a fixed order, so the result does not depend on
// scheduling.
template <typename T, int D_>
struct DirCCfg {
  static constexpr int D = D_;
  static constexpr int kThreads = 2 * D;
  static constexpr int kRowStride = D + ((sizeof(T) == 2) ? 2 : 1);   // odd number of 32-bit words
  static constexpr size_t kXBytes = (size_t)D * kRowStride * sizeof(T);
  static constexpr size_t kSmem = (size_t)D * D * 8 + kXBytes;
};

template <typename T, int D_>
__global__ void __launch_bounds__(2 * D_, D_ == 64 ? 3 : 1) dirc_kernel(
    const T* __restrict__ Q, const T* __restrict__ K, TensorLayout TL, int n, const TreeNode* __restrict__ nodes,
    int lvl_begin, int nodes_in_level, int npc, const double* __restrict__ M, const double* __restrict__ inv_s,
    const int* __restrict__ idx, int NI, double* __restrict__ zvec, double* __restrict__ wvec, uint64_t seed,
    int head_base, int power_iters, int tsel) {
  using Cfg = DirCCfg<T, D_>;
  constexpr int D = D_, RS = Cfg::kRowStride;
  constexpr int NT = Cfg::kThreads, HD = D / 2;   // threads, half length
  constexpr int NWD = D / 32;                     // warps holding one value per column
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* Ms = reinterpret_cast<double*>(smem_raw);             // D x D
  T* Xs = reinterpret_cast<T*>(smem_raw + (size_t)D * D * 8);   // D rows x RS
  __shared__ double red[2][D];
  __shared__ double zs[D], ws[D], xbar[D], fj[D], vs[D];
  __shared__ double qred[NWD][2];
  __shared__ double vred[2 * NWD];
  __shared__ int srow[D];
  const int th = tensor_head(blockIdx.y, tsel), bh = th >> 1, tensor = th & 1;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int ca = t & (D - 1), ch = t / D;       // column / half split
  const int rj = t >> 1, rh = t & 1;            // row / half split
  const T* X = (tensor == 0 ? Q : K) + TL.head(bh);
  {
    const double2* src = reinterpret_cast<const double2*>(M + (size_t)th * D * D);
    double2* dst = reinterpret_cast<double2*>(Ms);
#pragma unroll 4
    for (int e = t; e < D * D / 2; e += NT) dst[e] = src[e];
  }
  // w = M z (z in zs) into ws; returns (z . w, xbar . w) to every thread
  auto matvec = [&](double& zw, double& xw) {
    double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
    const int b0 = ch * HD;
#pragma unroll 4
    for (int b = 0; b < HD; b += 4) {
      a0 = fma(Ms[(b0 + b) * D + ca], zs[b0 + b], a0);
      a1 = fma(Ms[(b0 + b + 1) * D + ca], zs[b0 + b + 1], a1);
      a2 = fma(Ms[(b0 + b + 2) * D + ca], zs[b0 + b + 2], a2);
      a3 = fma(Ms[(b0 + b + 3) * D + ca], zs[b0 + b + 3], a3);
    }
    red[ch][ca] = (a0 + a1) + (a2 + a3);
    __syncthreads();
    if (t < D) {
      const double w = red[0][t] + red[1][t];
      ws[t] = w;
      double pz = zs[t] * w, px = xbar[t] * w;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        pz += __shfl_xor_sync(0xffffffffu, pz, o);
        px += __shfl_xor_sync(0xffffffffu, px, o);
      }
      if (lane == 0) { qred[warp][0] = pz; qred[warp][1] = px; }
    }
    __syncthreads();
    zw = 0.0; xw = 0.0;
#pragma unroll
    for (int q = 0; q < NWD; ++q) { zw += qred[q][0]; xw += qred[q][1]; }
  };
  const int first = blockIdx.x * npc, last = min(nodes_in_level, first + npc);
  for (int local = first; local < last; ++local) {
    const int node_id = lvl_begin + local;
    const TreeNode nd = nodes[node_id];
    const int m = min(D, nd.size);
    const uint64_t key = node_stream(seed, (uint64_t)(head_base + bh), (uint64_t)tensor, nd.heap);
    const uint64_t r = (nd.size > m) ? (splitmix64(key ^ kSampleTag) % (uint64_t)nd.size) : 0ull;
    __syncthreads();   // the previous node is done with every shared array
    if (t < D) {
      int row = 0;
      double sc = 0.0;
      if (t < m) {
        const int pos = (nd.size > m) ? (int)(((uint64_t)t * (uint64_t)nd.size + r) / (uint64_t)m) : t;
        row = idx ? idx[(size_t)th * n + nd.off + pos] : nd.off + pos;
        sc = (tensor == 0) ? inv_s[(size_t)bh * n + row] : 1.0;
      }
      srow[t] = row;
      vs[t] = sc;
    }
    __syncthreads();
    // stage the sample rows (rows >= m zero), 16-byte loads, 8 in flight
    {
      constexpr int VEC = 16 / (int)sizeof(T), CPR = D / VEC;   // chunks per row
      constexpr int WPR = RS * (int)sizeof(T) / 4;              // row stride in 32-bit words
      uint32_t* xw32 = reinterpret_cast<uint32_t*>(Xs);
#pragma unroll
      for (int u0 = 0; u0 < D * CPR; u0 += 8 * NT) {
        uint4 v4[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int e = u0 + u * NT + t;
          const int j = e / CPR, part = e % CPR;
          v4[u] = make_uint4(0, 0, 0, 0);
          if (e < D * CPR && j < m)
            v4[u] = *reinterpret_cast<const uint4*>(X + (size_t)srow[j] * TL.sn + part * VEC);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int e = u0 + u * NT + t;
          const int j = e / CPR, part = e % CPR;
          if (e < D * CPR) {
            uint32_t* dst = xw32 + (size_t)j * WPR + part * 4;
            dst[0] = v4[u].x; dst[1] = v4[u].y; dst[2] = v4[u].z; dst[3] = v4[u].w;
          }
        }
      }
    }
    __syncthreads();
    // d = 64: this thread's half row (for X w) and half column (for X^T v) of
    // the sample, converted to fp64 once per node instead of at every use (an
    // f32 -> f64 conversion issues at a quarter of the fp64 FMA rate); the
    // products below keep the same operands in the same order either way
    constexpr bool kRegX = D == 64;
    double xr_reg[kRegX ? HD : 1], xc_reg[kRegX ? HD : 1];
    if constexpr (kRegX) {
#pragma unroll
      for (int c = 0; c < HD; ++c) xr_reg[c] = (double)to_f(Xs[rj * RS + rh * HD + c]);
#pragma unroll
      for (int j = 0; j < HD; ++j) xc_reg[j] = (double)to_f(Xs[(ch * HD + j) * RS + ca]);
    }
    auto xcol = [&](int j) -> double {   // X[ch * HD + j][ca]
      if constexpr (kRegX) return xc_reg[j];
      else return (double)to_f(Xs[(ch * HD + j) * RS + ca]);
    };
    auto xrow = [&](int c) -> double {   // X[rj][rh * HD + c]
      if constexpr (kRegX) return xr_reg[c];
      else return (double)to_f(Xs[rj * RS + rh * HD + c]);
    };
    // sample mean
    {
      double a0 = 0.0, a1 = 0.0;
      const int j0 = ch * HD;
#pragma unroll
      for (int j = 0; j < HD; j += 2) {
        a0 = fma(vs[j0 + j], xcol(j), a0);
        a1 = fma(vs[j0 + j + 1], xcol(j + 1), a1);
      }
      red[ch][ca] = a0 + a1;
      __syncthreads();
      if (t < D) xbar[t] = (red[0][t] + red[1][t]) / (double)m;
    }
    // warm start from the Box-Muller normal g
    if (t < D) {
      const uint64_t ua = splitmix64(key + 2ull * t + 1ull);
      const uint64_t ub = splitmix64(key + 2ull * t + 2ull);
      const double u1 = (double)((ua >> 11) + 1ull) * 0x1.0p-53;
      const double u2 = (double)(ub >> 11) * 0x1.0p-53;
      zs[t] = sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
    }
    __syncthreads();
    double zw, xw;
    matvec(zw, xw);
    {
      const double gi = (zw > 0.0) ? 1.0 / sqrt(zw) : 0.0;
      if (t < D) {
        const double gh = zs[t] * gi;
        zs[t] = (nd.parent < 0) ? gh : 0.5 * (zvec[((size_t)th * NI + nd.parent) * D + t] + gh);
      }
    }
    __syncthreads();
    for (int it = 0; it < power_iters; ++it) {
      matvec(zw, xw);
      const double s = (zw > 0.0) ? 1.0 / sqrt(zw) : 0.0;
      // v_j = s (scale_j X_j . w - xbar . w): two threads per row
      double v = 0.0;
      {
        double d0 = 0.0, d1 = 0.0, d2 = 0.0, d3 = 0.0;
        const double* wr = ws + rh * HD;
#pragma unroll
        for (int c = 0; c < HD; c += 4) {
          d0 = fma(xrow(c), wr[c], d0);
          d1 = fma(xrow(c + 1), wr[c + 1], d1);
          d2 = fma(xrow(c + 2), wr[c + 2], d2);
          d3 = fma(xrow(c + 3), wr[c + 3], d3);
        }
        double d = (d0 + d1) + (d2 + d3);
        d += __shfl_xor_sync(0xffffffffu, d, 1);
        v = (rj < m) ? s * fma(vs[rj], d, -xw) : 0.0;
      }
      if (rh == 0) fj[rj] = v * vs[rj];
      double vsum = (rh == 0) ? v : 0.0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) vsum += __shfl_xor_sync(0xffffffffu, vsum, o);
      if (lane == 0) vred[warp] = vsum;
      __syncthreads();
      vsum = 0.0;
#pragma unroll
      for (int q = 0; q < 2 * NWD; ++q) vsum += vred[q];
      // z'_a = (sum_j v_j scale_j X_ja - xbar_a sum_j v_j) / m: two threads per column
      {
        double a0 = 0.0, a1 = 0.0;
        const int j0 = ch * HD;
#pragma unroll
        for (int j = 0; j < HD; j += 2) {
          a0 = fma(fj[j0 + j], xcol(j), a0);
          a1 = fma(fj[j0 + j + 1], xcol(j + 1), a1);
        }
        red[ch][ca] = a0 + a1;
      }
      __syncthreads();
      if (t < D) zs[t] = ((red[0][t] + red[1][t]) - xbar[t] * vsum) / (double)m;
      __syncthreads();
    }
    matvec(zw, xw);
    const double qi = (zw > 0.0) ? 1.0 / sqrt(zw) : 0.0;
    if (t < D) {
      const size_t o = ((size_t)th * NI + node_id) * D + t;
      zvec[o] = zs[t] * qi;
      wvec[o] = ws[t] * qi;
    }
  }
}

// ---------------------------------------------------------------------------
// K2a: projection key_i = x_i . w_node for every position of the level's
// internal nodes, stored as order-preserving uint64. A block covers
// kProjSpan consecutive positions, which meet at most kProjNodes nodes (every
// internal node holds more than c >= 64 vectors); their directions are staged
// in shared memory with a position -> node table. A group of G lanes reads
// one row (16 bytes per lane, coalesced); each group keeps kProjU rows in
// flight.
// ---------------------------------------------------------------------------
// d = 64 levels with at most this many nodes (over all tensor-heads) use the
// block-per-node power iteration
constexpr long long kDirCMaxNodes64 = 148 * 4;

constexpr int kProjSpan = 1024;
constexpr int kProjNodes = 20;   // > kProjSpan / 65 + 2, and at most 32 (one lane each)
constexpr int kProjU = 4;        // 8 measured slower (fewer blocks per SM)

template <typename T, int D>
__global__ void __launch_bounds__(256) project_kernel(const T* __restrict__ Q, const T* __restrict__ K,
                                                      TensorLayout TL, int n, const TreeNode* __restrict__ nodes,
                                                      int lb, int le, const double* __restrict__ inv_s,
                                                      const int* __restrict__ idx, int NI,
                                                      const double* __restrict__ wvec,
                                                      uint64_t* __restrict__ keys, int tsel) {
  constexpr int EPL = 16 / sizeof(T);        // elements per lane (16 bytes)
  constexpr int G = D / EPL;                 // lanes per row
  constexpr int RPW = 32 / G;                // rows per warp step
  constexpr int STEP = 8 * RPW;              // rows per block step (8 warps)
  __shared__ double ws[kProjNodes][D];
  __shared__ int n_off[kProjNodes], n_end[kProjNodes], n_id[kProjNodes];
  __shared__ unsigned char slot_of[kProjSpan];
  __shared__ int rows_s[kProjSpan];      // source row of each position
  __shared__ int s_cnt;
  const int th = tensor_head(blockIdx.y, tsel), bh = th >> 1, tensor = th & 1;
  const T* X = (tensor == 0 ? Q : K) + TL.head(bh);
  const int base = blockIdx.x * kProjSpan;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp == 0) {
    // last node with off <= base (32-ary search), lb - 1 if none
    int lo = lb, hi = le, f = lb - 1;
    while (hi > lo) {
      const int step = (hi - lo + 31) / 32;
      const int probe = lo + lane * step;
      const bool ok = probe < hi && nodes[probe].off <= base;
      const unsigned b = __ballot_sync(0xffffffffu, ok);
      if (b == 0) break;
      const int L = 31 - __clz(b);
      f = lo + L * step;
      if (step == 1) break;
      lo = f;
      hi = min(hi, f + step);
    }
    const int start = f < lb ? lb : f;
    const int i = start + lane;
    bool take = false;
    int off = 0, end = 0;
    if (lane < kProjNodes && i < le) {
      off = nodes[i].off;
      end = off + nodes[i].size;
      take = off < base + kProjSpan && end > base;
    }
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int sl = __popc(tb & ((1u << lane) - 1u));
      n_off[sl] = off; n_end[sl] = end; n_id[sl] = i;
    }
    if (lane == 0) s_cnt = __popc(tb);
  }
  __syncthreads();
  const int cnt = s_cnt;
  // node slot of each position of the span and, for the positions inside a
  // node of this level (only those: elsewhere the index buffer holds nothing
  // meaningful), the source row, all of a thread's index loads in flight
  {
    unsigned char sl[kProjSpan / 256];
    int rv[kProjSpan / 256];
#pragma unroll
    for (int u = 0; u < kProjSpan / 256; ++u) {
      const int pos = base + u * 256 + threadIdx.x;
      sl[u] = 255;
      for (int q = 0; q < cnt; ++q)
        if (pos >= n_off[q] && pos < n_end[q]) sl[u] = (unsigned char)q;
      slot_of[u * 256 + threadIdx.x] = sl[u];
      rv[u] = 0;
      if (sl[u] != 255) rv[u] = idx ? idx[(size_t)th * n + pos] : pos;
    }
#pragma unroll
    for (int u = 0; u < kProjSpan / 256; ++u) rows_s[u * 256 + threadIdx.x] = rv[u];
  }
  for (int e = threadIdx.x; e < cnt * D; e += 256)
    ws[e / D][e % D] = wvec[((size_t)th * NI + n_id[e / D]) * D + (e % D)];
  __syncthreads();
  const int sub = lane / G, gl = lane % G;
  // this lane's EPL direction values of the current node, reloaded only when
  // the node changes (rows are in position order, so rarely)
  int wslot = -1;
  double wr[EPL];
#pragma unroll
  for (int q = 0; q < EPL; ++q) wr[q] = 0.0;
  for (int r0 = warp * RPW + sub; r0 < kProjSpan; r0 += STEP * kProjU) {
    int slot[kProjU], row[kProjU];
    uint4 raw[kProjU];
    double sc[kProjU];
#pragma unroll
    for (int u = 0; u < kProjU; ++u) {
      const int rr = r0 + u * STEP;
      const int pos = base + rr;
      slot[u] = (rr < kProjSpan && pos < n) ? slot_of[rr] : 255;
      row[u] = 0;
      if (slot[u] != 255) row[u] = rows_s[rr];
    }
#pragma unroll
    for (int u = 0; u < kProjU; ++u) {
      raw[u] = make_uint4(0, 0, 0, 0);
      sc[u] = 1.0;
      if (slot[u] != 255) {
        raw[u] = *reinterpret_cast<const uint4*>(X + (size_t)row[u] * TL.sn + gl * EPL);
        if (tensor == 0) sc[u] = inv_s[(size_t)bh * n + row[u]];
      }
    }
#pragma unroll
    for (int u = 0; u < kProjU; ++u) {
      double s = 0.0;
      if (slot[u] != 255) {
        if (slot[u] != wslot) {
          wslot = slot[u];
#pragma unroll
          for (int q = 0; q < EPL; ++q) wr[q] = ws[wslot][gl * EPL + q];
        }
        const T* e = reinterpret_cast<const T*>(&raw[u]);
        double s0 = 0.0, s1 = 0.0;
#pragma unroll
        for (int q = 0; q < EPL; q += 2) {
          s0 = fma((double)to_f(e[q]), wr[q], s0);
          s1 = fma((double)to_f(e[q + 1]), wr[q + 1], s1);
        }
        s = s0 + s1;
      }
#pragma unroll
      for (int o = G / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (slot[u] != 255 && gl == 0) keys[(size_t)th * n + base + r0 + u * STEP] = ordered_key(s * sc[u]);
    }
  }
}

// Random-cluster baseline: the key of every position is the counter-based
// hash of its token, the same at every level, so the splits cut the fixed
// random order of the tokens into groups of c (remainder last). Positions
// outside this level's nodes get a key too; nothing reads it.
__global__ void __launch_bounds__(256) hash_keys_kernel(int n, const int* __restrict__ idx, uint64_t seed,
                                                        int head_base, uint64_t* __restrict__ keys, int tsel) {
  const int th = tensor_head(blockIdx.y, tsel), bh = th >> 1, tensor = th & 1;
  const int pos = blockIdx.x * 256 + threadIdx.x;
  if (pos >= n) return;
  const int row = idx ? idx[(size_t)th * n + pos] : pos;
  keys[(size_t)th * n + pos] =
      splitmix64(node_stream(seed, (uint64_t)(head_base + bh), (uint64_t)tensor, 0ull) ^ (uint64_t)(uint32_t)row);
}

// ---------------------------------------------------------------------------
// K2b: the t-th smallest key of a node (MSD radix select, 8-bit digits).
// Nodes of at most kSelCap keys are read into shared memory once; larger
// nodes are scanned in global memory until the candidates sharing the
// selected prefix fit. Output: the threshold key T and eq_left = how many
// keys equal to T go below the split (the first ones in row order, so equal
// projections are ordered by row index).
// ---------------------------------------------------------------------------
struct SelectResult { uint64_t T; int eq_left; int pad; };
constexpr int kSelCap = 8192;
constexpr int kSelU = 4;   // keys per thread in flight in the global passes (16 measured the same)

template <int NT>
__global__ void __launch_bounds__(NT) select_kernel(const TreeNode* __restrict__ nodes, int lb,
                                                    int nodes_in_level, int n,
                                                    const uint64_t* __restrict__ keys,
                                                    SelectResult* __restrict__ sel, int tsel) {
  __shared__ unsigned int hist[256];
  __shared__ int s_digit, s_rank, s_cnt, s_ncand;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem_raw);   // kSelCap keys
  const int th = tensor_head(blockIdx.y, tsel);
  const TreeNode nd = nodes[lb + blockIdx.x];
  const uint64_t* base = keys + (size_t)th * n + nd.off;
  const int size = nd.size;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int rank = nd.t - 1;
  uint64_t prefix = 0, mask = 0;
  bool global_mode = size > kSelCap;
  int ncand = size;
  if (!global_mode) {
    for (int i = threadIdx.x; i < size; i += NT) cand[i] = base[i];
  }
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += NT) hist[i] = 0;
    __syncthreads();
    const int cnt_total = global_mode ? size : ncand;
    // warp-aggregated histogram increment of one key
    auto count = [&](bool ok, uint64_t k) {
      const unsigned dg = (unsigned)((k >> shift) & 0xFF);
      const unsigned act = __ballot_sync(0xffffffffu, ok);
      if (ok) {
        const unsigned peers = __match_any_sync(act, dg);
        if ((__ffs(peers) - 1) == lane) atomicAdd(&hist[dg], (unsigned)__popc(peers));
      }
    };
    if (global_mode) {
      // kSelU keys per thread per step, their loads in flight together
      for (int i0 = 0; i0 < cnt_total; i0 += NT * kSelU) {
        uint64_t kk[kSelU];
#pragma unroll
        for (int u = 0; u < kSelU; ++u) {
          const int i = i0 + u * NT + threadIdx.x;
          kk[u] = i < cnt_total ? base[i] : 0ull;
        }
#pragma unroll
        for (int u = 0; u < kSelU; ++u)
          count(i0 + u * NT + (int)threadIdx.x < cnt_total && (kk[u] & mask) == prefix, kk[u]);
      }
    } else {
      for (int i0 = 0; i0 < cnt_total; i0 += NT) {
        const int i = i0 + threadIdx.x;
        const uint64_t k = i < cnt_total ? cand[i] : 0ull;
        count(i < cnt_total && (k & mask) == prefix, k);
      }
    }
    __syncthreads();
    if (warp == 0) {
      // digit holding the rank: lane L owns bins 8L..8L+7
      unsigned h[8], local = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) { h[q] = hist[lane * 8 + q]; local += h[q]; }
      unsigned incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned excl = incl - local;
      const bool mine = excl <= (unsigned)rank && (unsigned)rank < incl;
      if (mine) {
        unsigned r = (unsigned)rank - excl;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (r < h[q]) { s_digit = lane * 8 + q; s_rank = (int)r; s_cnt = (int)h[q]; break; }
          r -= h[q];
        }
      }
    }
    __syncthreads();
    rank = s_rank;
    prefix |= (uint64_t)s_digit << shift;
    mask |= (uint64_t)0xFF << shift;
    const int cnt = s_cnt;
    __syncthreads();
    if (shift > 0 && cnt <= kSelCap && (global_mode || cnt < ncand)) {
      // keep only the candidates that share the prefix
      if (threadIdx.x == 0) s_ncand = 0;
      __syncthreads();
      if (global_mode) {
        for (int i0 = 0; i0 < size; i0 += NT * kSelU) {
          uint64_t kk[kSelU];
#pragma unroll
          for (int u = 0; u < kSelU; ++u) {
            const int i = i0 + u * NT + threadIdx.x;
            kk[u] = i < size ? base[i] : ~prefix;   // ~prefix never matches (the mask is not empty)
          }
#pragma unroll
          for (int u = 0; u < kSelU; ++u)
            if ((kk[u] & mask) == prefix) cand[atomicAdd(&s_ncand, 1)] = kk[u];
        }
      } else {
        // in place: read all candidates first, then write the survivors
        uint64_t mine[kSelCap / NT];
        int nm = 0;
        for (int i = threadIdx.x; i < ncand; i += NT) {
          const uint64_t k = cand[i];
          if ((k & mask) == prefix) mine[nm++] = k;
        }
        __syncthreads();
        for (int q = 0; q < nm; ++q) cand[atomicAdd(&s_ncand, 1)] = mine[q];
      }
      __syncthreads();
      ncand = s_ncand;
      global_mode = false;
      __syncthreads();
    }
  }
  if (threadIdx.x == 0) {
    SelectResult r;
    r.T = prefix; r.eq_left = rank + 1; r.pad = 0;
    sel[(size_t)th * nodes_in_level + blockIdx.x] = r;
  }
}

// ---------------------------------------------------------------------------
// K2c: stable partition, two passes over node-aligned chunks.
// Pass A counts keys below / equal to T per chunk; pass B scans and scatters
// row indices to the children (a child that is a leaf writes straight into
// the cluster permutation).
// ---------------------------------------------------------------------------
constexpr int kPartThreads = 256;
constexpr int kPartPer = kPartChunk / kPartThreads;   // 8 positions per thread

__global__ void __launch_bounds__(kPartThreads) part_count_kernel(
    const TreeNode* __restrict__ nodes, int lb, int nodes_in_level, int n, int pch,
    const uint64_t* __restrict__ keys, const SelectResult* __restrict__ sel, int2* __restrict__ cnt, int tsel) {
  const int th = tensor_head(blockIdx.z, tsel), nl = blockIdx.y, ch = blockIdx.x;
  const TreeNode nd = nodes[lb + nl];
  const SelectResult sr = sel[(size_t)th * nodes_in_level + nl];
  const int p0 = ch * kPartChunk, p1 = min(nd.size, p0 + kPartChunk);
  int less = 0, eq = 0;
  for (int p = p0 + threadIdx.x; p < p1; p += kPartThreads) {
    const uint64_t k = keys[(size_t)th * n + nd.off + p];
    less += (k < sr.T);
    eq += (k == sr.T);
  }
  __shared__ int rl[kPartThreads / 32], re[kPartThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    less += __shfl_xor_sync(0xffffffffu, less, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  if ((threadIdx.x & 31) == 0) { rl[threadIdx.x >> 5] = less; re[threadIdx.x >> 5] = eq; }
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0, b = 0;
    for (int i = 0; i < kPartThreads / 32; ++i) { a += rl[i]; b += re[i]; }
    cnt[((size_t)th * nodes_in_level + nl) * pch + ch] = make_int2(a, b);
  }
}

// Block-wide exclusive scan of one int per thread (256 threads).
__device__ __forceinline__ int block_excl_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    int s = 0;
    for (int i = 0; i < kPartThreads / 32; ++i) { const int t = warp_tot[i]; warp_tot[i] = s; s += t; }
    *total = s;
  }
  __syncthreads();
  const int r = warp_tot[warp] + x - v;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kPartThreads) part_scatter_kernel(
    const TreeNode* __restrict__ nodes, int lb, int nodes_in_level, int n, int c, int pch,
    const uint64_t* __restrict__ keys, const SelectResult* __restrict__ sel,
    const int2* __restrict__ cnt, const int* __restrict__ idx_in, int* __restrict__ idx_out,
    int32_t* __restrict__ perm_q, int32_t* __restrict__ perm_k, int Cc, int tsel) {
  __shared__ int warp_tot[kPartThreads / 32];
  __shared__ int total;
  const int th = tensor_head(blockIdx.z, tsel), nl = blockIdx.y, ch = blockIdx.x;
  const int bh = th >> 1, tensor = th & 1;
  const TreeNode nd = nodes[lb + nl];
  const int p0 = ch * kPartChunk;
  if (p0 >= nd.size) return;
  const SelectResult sr = sel[(size_t)th * nodes_in_level + nl];
  const int2* cn = cnt + ((size_t)th * nodes_in_level + nl) * pch;
  int less_before = 0, eq_before = 0;
  for (int i = 0; i < ch; ++i) { less_before += cn[i].x; eq_before += cn[i].y; }
  const int left_before = less_before + min(eq_before, sr.eq_left);
  // this thread's positions: p0 + threadIdx.x * kPartPer + q
  uint64_t kv[kPartPer];
  int eq_local = 0;
#pragma unroll
  for (int q = 0; q < kPartPer; ++q) {
    const int p = p0 + threadIdx.x * kPartPer + q;
    kv[q] = (p < nd.size) ? keys[(size_t)th * n + nd.off + p] : ~0ull;
    eq_local += (p < nd.size) && (kv[q] == sr.T);
  }
  const int eq_excl = block_excl_scan(eq_local, warp_tot, &total);
  bool goes_left[kPartPer];
  int left_local = 0;
  {
    int er = eq_before + eq_excl;
#pragma unroll
    for (int q = 0; q < kPartPer; ++q) {
      const int p = p0 + threadIdx.x * kPartPer + q;
      bool gl = false;
      if (p < nd.size) {
        if (kv[q] < sr.T) gl = true;
        else if (kv[q] == sr.T) { gl = (er < sr.eq_left); ++er; }
      }
      goes_left[q] = gl;
      left_local += gl;
    }
  }
  const int left_excl = block_excl_scan(left_local, warp_tot, &total);
  const int t = nd.t;
  const bool left_leaf = (t <= c), right_leaf = (nd.size - t <= c);
  int32_t* perm = (tensor == 0 ? perm_q : perm_k) + (size_t)bh * Cc;
  int lrank = left_before + left_excl;
#pragma unroll
  for (int q = 0; q < kPartPer; ++q) {
    const int p = p0 + threadIdx.x * kPartPer + q;
    if (p >= nd.size) break;
    const int row = idx_in ? idx_in[(size_t)th * n + nd.off + p] : nd.off + p;
    if (goes_left[q]) {
      const int dst = nd.off + lrank;
      if (left_leaf) perm[dst] = row; else idx_out[(size_t)th * n + dst] = row;
      ++lrank;
    } else {
      const int dst = nd.off + t + (p - lrank);
      if (right_leaf) perm[dst] = row; else idx_out[(size_t)th * n + dst] = row;
    }
  }
}

// ---------------------------------------------------------------------------
// S5: counts, pad slots and centroids (fp64 means of the members' original
// vectors, eq. 18). levels == 0 means the single cluster holds every token.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256) centroid_kernel(const T* __restrict__ Q, const T* __restrict__ K,
                                                       TensorLayout TL, int n, int c, int C, int levels,
                                                       int32_t* __restrict__ perm_q, int32_t* __restrict__ perm_k,
                                                       int32_t* __restrict__ count_q, int32_t* __restrict__ count_k,
                                                       double* __restrict__ qbar, double* __restrict__ kbar,
                                                       int tsel) {
  constexpr int RG = 256 / D;
  const int a = blockIdx.x, th = tensor_head(blockIdx.y, tsel), bh = th >> 1, tensor = th & 1;
  const int cnt = (a < C - 1) ? c : n - (C - 1) * c;
  int32_t* perm = (tensor == 0 ? perm_q : perm_k) + (size_t)bh * C * c + (size_t)a * c;
  if (levels == 0) {
    for (int j = threadIdx.x; j < cnt; j += 256) perm[j] = j;
    __syncthreads();
  }
  for (int j = cnt + threadIdx.x; j < c; j += 256) perm[j] = -1;
  if (threadIdx.x == 0) ((tensor == 0) ? count_q : count_k)[(size_t)bh * C + a] = cnt;
  const T* X = (tensor == 0 ? Q : K) + TL.head(bh);
  const int col = threadIdx.x % D, rg = threadIdx.x / D;
  // members rg, rg + RG, ... summed in that order, four row loads in flight
  double s = 0.0;
  int j = rg;
  for (; j + 3 * RG < cnt; j += 4 * RG) {
    int r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) r[u] = (levels == 0) ? j + u * RG : perm[j + u * RG];
    T x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = X[(size_t)r[u] * TL.sn + col];
#pragma unroll
    for (int u = 0; u < 4; ++u) s += (double)to_f(x[u]);
  }
  for (; j < cnt; j += RG) {
    const int row = (levels == 0) ? j : perm[j];
    s += (double)to_f(X[(size_t)row * TL.sn + col]);
  }
  __shared__ double red[256];
  red[threadIdx.x] = s;
  __syncthreads();
  if (rg == 0) {
    double t = 0.0;
    for (int g = 0; g < RG; ++g) t += red[g * D + col];
    ((tensor == 0) ? qbar : kbar)[((size_t)bh * C + a) * D + col] = t / (double)cnt;
  }
}

template <typename T, int D>
cudaError_t run_cluster(const T* Q, const T* K, const ca_shape* s, const ca_cluster_params* p,
                        const ca_clusters* out, const TreePlan& plan, const TreePlan& plan_k, const ClusterWs& L,
                        char* ws, cudaStream_t st) {
  const int n = s->n_valid;
  const TensorLayout TL = tensor_layout(s);
  const int BH = L.BH, TH = L.TH, NI = L.NI;
  const int nch = L.nch;
  // Queries and keys share one tree when their cluster sizes are equal; with
  // unequal sizes each tensor walks its own (its nodes in their own table).
  const bool same_tree = key_c(s) == s->c;
  TreeNode* nodes_t[2] = {reinterpret_cast<TreeNode*>(ws + L.nodes), reinterpret_cast<TreeNode*>(ws + L.nodes_k)};
  int* level_begin_t[2] = {reinterpret_cast<int*>(ws + L.level_begin), reinterpret_cast<int*>(ws + L.level_begin_k)};
  double* M = reinterpret_cast<double*>(ws + L.M);
  double* colpart = reinterpret_cast<double*>(ws + L.colsum_part);
  double* metpart = reinterpret_cast<double*>(ws + L.met_part);
  double* inv_s = reinterpret_cast<double*>(ws + L.inv_s);
  int* idxbuf[2] = {reinterpret_cast<int*>(ws + L.idx0), reinterpret_cast<int*>(ws + L.idx1)};
  uint64_t* keys = reinterpret_cast<uint64_t*>(ws + L.keys);
  double* zvec = reinterpret_cast<double*>(ws + L.zvec);
  double* wvec = reinterpret_cast<double*>(ws + L.wvec);
  SelectResult* sel = reinterpret_cast<SelectResult*>(ws + L.sel);
  int2* ccnt = reinterpret_cast<int2*>(ws + L.chunk_cnt);
  const int power_iters = p->power_iters > 0 ? p->power_iters : 8;
  const int sample_factor = p->sample_factor > 0 ? p->sample_factor : 1;
  const int transform = p->transform;
  // queries are divided by |R_k q| only in the top-k form (eq. 16); the
  // adaptive form (eq. 15) and the untransformed ablation use scale 1
  const int normalize = transform && p->query_form == 0;

  const bool random_clusters = p->method == 1;
  const bool diagonal = p->method == 2;
  double* basis = reinterpret_cast<double*>(ws + L.basis);
  const bool any_split = plan.levels > 0 || plan_k.levels > 0;
  if (any_split) {
    plan_kernel<<<1, 1024, 0, st>>>(n, s->c, nodes_t[0], level_begin_t[0]);
    if (!same_tree) plan_kernel<<<1, 1024, 0, st>>>(n, key_c(s), nodes_t[1], level_begin_t[1]);
    if (!random_clusters) {
      colsum_kernel<T, D><<<dim3(nch, BH), 256, 0, st>>>(K, TL, n, colpart);
      const size_t syrk_smem = SyrkCfg<D>::template smem<T>();
      const size_t mma_smem = SyrkMmaCfg<D>::template smem<T>();
      cudaFuncSetAttribute(syrk_mma_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mma_smem);
      syrk_mma_kernel<T, D><<<dim3(nch, BH, 2), SyrkMmaCfg<D>::kThreads, mma_smem, st>>>(Q, K, TL, n, nch,
                                                                                        colpart, metpart);
      metric_reduce_kernel<D><<<dim3(D * D / 256, TH), 256, 0, st>>>(metpart, nch, n, transform, M);
      if (D == 64 && normalize) {
        qnorm64_kernel<T><<<dim3((n + 127) / 128, BH), 128, 0, st>>>(Q, TL, n, M, inv_s);
      } else {
        const size_t qn_smem = (size_t)D * D * 8 + (size_t)128 * (D + 1) * 4;
        cudaFuncSetAttribute(qnorm_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)qn_smem);
        qnorm_kernel<T, D><<<dim3((n + 127) / 128, BH), 256, qn_smem, st>>>(Q, TL, n, M, normalize, inv_s);
      }
      if (diagonal) {
        // covariance of the scaled query rows (weights 1 / |R_k q| in the
        // top-k form, 1 otherwise): weighted column sums into the key sums'
        // buffer and the centred weighted Gram into the queries' slot of the
        // partials, both free once M and the query scales exist
        colsum_kernel<T, D, true><<<dim3(nch, BH), 256, 0, st>>>(Q, TL, n, colpart, inv_s);
        cudaFuncSetAttribute(syrk_kernel<T, D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)syrk_smem);
        syrk_kernel<T, D, true><<<dim3(nch, BH, 1), SyrkCfg<D>::kThreads, syrk_smem, st>>>(
            Q, K, TL, n, nch, colpart, metpart, inv_s);
        const cudaError_t e = launch_diag_basis(D, TH, BH, nch, n, metpart, M,
                                                reinterpret_cast<double*>(ws + L.cov),
                                                reinterpret_cast<double*>(ws + L.basis_scratch), basis, st);
        if (e != cudaSuccess) return e;
      }
    }
  }
  const int m_cap = sample_factor * D;
  const int dir_warps = DirCfg<T, D>::warps(m_cap);
  const size_t dir_smem = (size_t)D * D * 8 + (size_t)dir_warps * DirCfg<T, D>::warp_bytes(m_cap);
  cudaFuncSetAttribute(dir_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dir_smem);
  cudaFuncSetAttribute(dirc_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DirCCfg<T, D>::kSmem);
  cudaFuncSetAttribute(select_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelCap * 8);
  cudaFuncSetAttribute(select_kernel<1024>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelCap * 8);
  // The levels of one tree, for both tensors (tsel < 0) or one (tsel = 0, 1);
  // then the centroids of the clusters that tree makes.
  auto run_tree = [&](const TreePlan& pl, int tsel) -> cudaError_t {
    const int c = tsel == 1 ? key_c(s) : s->c, C = pl.C;
    const int rows = tsel < 0 ? TH : BH;   // grid rows: tensor-heads
    TreeNode* nodes = nodes_t[tsel == 1 ? 1 : 0];
    for (int l = 0; l < pl.levels; ++l) {
      const int lb = pl.level_begin[l], le = pl.level_begin[l + 1], nl = le - lb;
      const int* idx_in = (l == 0) ? nullptr : idxbuf[l & 1];
      int* idx_out = idxbuf[(l + 1) & 1];
      if (random_clusters) {
        hash_keys_kernel<<<dim3((n + 255) / 256, rows), 256, 0, st>>>(n, idx_in, p->seed, p->head_base, keys, tsel);
      } else if (diagonal) {
        const cudaError_t e = launch_diag_dir<T, D>(Q, K, TL, n, nodes, lb, nl, rows, basis, inv_s, idx_in,
                                                    NI, wvec, p->seed, p->head_base, tsel, st);
        if (e != cudaSuccess) return e;
      } else if (sample_factor == 1 && (D == 128 || (long long)nl * rows <= kDirCMaxNodes64)) {
        // a block per node: d = 128, or d = 64 levels with few nodes (about
        // four blocks per SM over the whole level)
        const int npc = (int)(((long long)nl * rows + 4 * 148 - 1) / (4 * 148));
        dirc_kernel<T, D><<<dim3((nl + npc - 1) / npc, rows), DirCCfg<T, D>::kThreads, DirCCfg<T, D>::kSmem, st>>>(
            Q, K, TL, n, nodes, lb, nl, npc, M, inv_s, idx_in, NI, zvec, wvec, p->seed, p->head_base,
            power_iters, tsel);
      } else {
        dir_kernel<T, D><<<dim3((nl + dir_warps - 1) / dir_warps, rows), dir_warps * 32, dir_smem, st>>>(
            Q, K, TL, n, nodes, lb, nl, M, inv_s, idx_in, NI, zvec, wvec, p->seed, p->head_base, power_iters,
            sample_factor, tsel);
      }
      if (!random_clusters)
        project_kernel<T, D><<<dim3((n + kProjSpan - 1) / kProjSpan, rows), 256, 0, st>>>(
            Q, K, TL, n, nodes, lb, le, inv_s, idx_in, NI, wvec, keys, tsel);
      if (pl.level_max_size[l] <= kSelCap)   // candidates buffer sized to the level's largest node
        select_kernel<256><<<dim3(nl, rows), 256, (size_t)pl.level_max_size[l] * 8, st>>>(nodes, lb, nl, n, keys,
                                                                                        sel, tsel);
      else
        select_kernel<1024><<<dim3(nl, rows), 1024, kSelCap * 8, st>>>(nodes, lb, nl, n, keys, sel, tsel);
      const int pch = (pl.level_max_size[l] + kPartChunk - 1) / kPartChunk;
      part_count_kernel<<<dim3(pch, nl, rows), kPartThreads, 0, st>>>(nodes, lb, nl, n, pch, keys, sel, ccnt, tsel);
      part_scatter_kernel<<<dim3(pch, nl, rows), kPartThreads, 0, st>>>(nodes, lb, nl, n, c, pch, keys, sel,
                                                                      ccnt, idx_in, idx_out, out->perm_q,
                                                                      out->perm_k, C * c, tsel);
    }
    centroid_kernel<T, D><<<dim3(C, rows), 256, 0, st>>>(Q, K, TL, n, c, C, pl.levels, out->perm_q,
                                                         out->perm_k, out->count_q, out->count_k, out->qbar,
                                                         out->kbar, tsel);
    return cudaGetLastError();
  };
  cudaError_t e;
  if (same_tree) {
    e = run_tree(plan, -1);
  } else {
    e = run_tree(plan, 0);
    if (e == cudaSuccess) e = run_tree(plan_k, 1);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool host_plan(int n, int c, TreePlan* plan) {
  plan->n = n; plan->c = c; plan->C = (n + c - 1) / c;
  plan->internal = plan->C - 1;
  TreeNode* nodes = new TreeNode[plan->internal > 0 ? plan->internal : 1];
  int lb[kMaxLevels + 1];
  const int L = plan_tree(n, c, nodes, lb, kMaxLevels);
  bool ok = true;
  if (L >= kMaxLevels) ok = false;
  plan->levels = L;
  for (int l = 0; l <= L && l <= kMaxLevels; ++l) plan->level_begin[l] = lb[l];
  for (int l = 0; l < L && l < kMaxLevels; ++l) {
    int mx = 0;
    for (int i = lb[l]; i < lb[l + 1]; ++i) mx = nodes[i].size > mx ? nodes[i].size : mx;
    plan->level_max_size[l] = mx;
  }
  if (L > 0 && lb[L] != plan->internal) ok = false;
  delete[] nodes;
  return ok;
}

bool cluster_ws_layout(const ca_shape* s, const TreePlan& plan, const TreePlan& plan_k, ClusterWs* w) {
  const size_t n = s->n_valid, d = s->d;
  const size_t BH = (size_t)s->B * s->H, TH = 2 * BH;
  const int ni = plan.internal > plan_k.internal ? plan.internal : plan_k.internal;
  const size_t NI = ni > 0 ? (size_t)ni : 1;
  w->BH = (int)BH; w->TH = (int)TH; w->NI = (int)NI;
  w->nch = (int)((n + kMetricChunk - 1) / kMetricChunk);
  int pmax = 1;
  size_t chunk_cnt = 1;
  for (const TreePlan* pl : {&plan, &plan_k}) {
    for (int l = 0; l < pl->levels; ++l) {
      const int pch = (pl->level_max_size[l] + kPartChunk - 1) / kPartChunk;
      const int nl = pl->level_begin[l + 1] - pl->level_begin[l];
      pmax = pch > pmax ? pch : pmax;
      const size_t need = (size_t)nl * pch;
      chunk_cnt = need > chunk_cnt ? need : chunk_cnt;
    }
  }
  w->pch_max = pmax;
  const size_t NIq = plan.internal > 0 ? (size_t)plan.internal : 1;
  const size_t NIk = plan_k.internal > 0 ? (size_t)plan_k.internal : 1;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = align_up(o + bytes); return r; };
  w->nodes = take(NIq * sizeof(TreeNode));
  w->level_begin = take((kMaxLevels + 1) * sizeof(int));
  w->nodes_k = take(NIk * sizeof(TreeNode));
  w->level_begin_k = take((kMaxLevels + 1) * sizeof(int));
  w->M = take(TH * d * d * 8);
  w->kmean = take(BH * d * 8);
  w->colsum_part = take(BH * w->nch * d * 8);
  w->met_part = take(BH * 2 * w->nch * d * d * 8);
  w->inv_s = take(BH * n * 8);
  w->idx0 = take(TH * n * 4);
  w->idx1 = take(TH * n * 4);
  w->keys = take(TH * n * 8);
  w->zvec = take(TH * NI * d * 8);
  w->wvec = take(TH * NI * d * 8);
  w->sel = take(TH * NI * 16);
  w->chunk_cnt = take(TH * chunk_cnt * 8);
  w->cov = take(TH * d * d * 8);
  w->basis = take(TH * d * d * 8);
  w->basis_scratch = take(TH * 2 * d * d * 8);
  w->total = o;
  return true;
}

cudaError_t launch_cluster(const void* Q, const void* K, const ca_shape* s, const ca_cluster_params* p,
                           const ca_clusters* out, const TreePlan& plan, const TreePlan& plan_k, const ClusterWs& L,
                           char* ws, cudaStream_t st) {
  if (s->dtype == CA_BF16) {
    using T = __nv_bfloat16;
    if (s->d == 64) return run_cluster<T, 64>((const T*)Q, (const T*)K, s, p, out, plan, plan_k, L, ws, st);
    return run_cluster<T, 128>((const T*)Q, (const T*)K, s, p, out, plan, plan_k, L, ws, st);
  }
  using T = float;
  if (s->d == 64) return run_cluster<T, 64>((const T*)Q, (const T*)K, s, p, out, plan, plan_k, L, ws, st);
  return run_cluster<T, 128>((const T*)Q, (const T*)K, s, p, out, plan, plan_k, L, ws, st);
}

}  // namespace ca
