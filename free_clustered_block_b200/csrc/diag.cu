// Diagonalized recursive splitting ("ClusterAttention", Section 3.2.1
// "Diagonalized recursive splitting"; complexity in Appendix D.2, eq. 53-54).
//
// Instead of a power iteration per set, the representations of the full set
// are rotated once into their principal-component basis and every set is
// split on the coordinate with the highest variance in its sample.
//
// With y = R x the representation of a raw row x (R the symmetric root of the
// metric, eq. 13-14; queries in the top-k form also scaled by 1 / |R_k q|,
// eq. 16), the covariance of the representations is R C R, where C is the
// covariance of the (scaled) raw rows. Its unit eigenvectors u_j, ordered by
// descending eigenvalue, give coordinate j of a row as y . u_j = x . w_j with
// w_j = R u_j, each signed so that w_j's entry of largest magnitude is
// positive. The rotation is therefore never materialised: the per-set
// kernel evaluates the sample's coordinates through the w_j, picks the
// coordinate of highest sample variance, and hands w_j to the projection
// kernel shared with the basic splitting (which multiplies the query scale).
//
// Kernels:
//   cov_reduce_kernel   chunk partials -> C per tensor-head (fp64)
//   diag_basis_kernel   one CTA per tensor-head: pivoted Cholesky factor F of
//                       the metric, F^T C F, Jacobi eigensolver, W = (F U')^T
//   diag_dir_kernel     per set: sample coordinates, variances, argmax, w_j*
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ca_internal.cuh"

namespace ca {
namespace {

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// ---------------------------------------------------------------------------
// C[th] = (sum of the chunk partials) / n. Tensor-head th = 2 bh + tensor reads
// slot z = tensor of the Gram partials: z = 0 holds the weighted, centred
// query rows, z = 1 the centred key rows.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) cov_reduce_kernel(const double* __restrict__ part, int nch, int n,
                                                         double* __restrict__ C) {
  const int th = blockIdx.y, bh = th >> 1, tensor = th & 1;
  const double* p = part + ((size_t)bh * 2 + tensor) * nch * D * D;
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e >= D * D) return;
  double v = 0.0;
  for (int ch = 0; ch < nch; ++ch) v += p[(size_t)ch * D * D + e];
  C[(size_t)th * D * D + e] = v / (double)n;
}

// ---------------------------------------------------------------------------
// Symmetric eigensolver: cyclic Jacobi (Golub & Van Loan, "Matrix
// Computations", Section 8.5, the symmetric Schur decomposition of 2 x 2
// blocks) with the round-robin ("circle") ordering, under which the D / 2
// rotations of one step touch disjoint index pairs and are applied together:
// every 2 x 2 block of A between pairs k and l becomes J_k^T B J_l.
// A is kept packed (upper triangle, row-major) in shared memory; the
// eigenvectors accumulate as the rows of Vt (Vt[k][i] = V[i][k]).
// A rotation is skipped when |a_pq| <= eps sqrt(|a_pp a_qq|); the solver stops
// after a sweep without rotations (at most kJacobiMaxSweeps sweeps).
// ---------------------------------------------------------------------------
constexpr int kJacobiMaxSweeps = 40;
constexpr double kJacobiEps = 2.220446049250313e-16;   // 2^-52

template <int D>
struct BasisCfg {
  static constexpr int kThreads = 512;   // 16 warps: each step's latency spread over more schedulers
  static constexpr int P = D / 2;                       // pairs per step
  static constexpr int kPacked = D * (D + 1) / 2;
  static constexpr int kBlocks = P * (P + 1) / 2;       // pair blocks (k <= l)
  static constexpr size_t kSmem = (size_t)kPacked * 8 + (size_t)D * D * 8 + (size_t)kBlocks * 4;
};

template <int D>
__device__ __forceinline__ int packed(int i, int j) {   // i <= j
  return i * (2 * D - i + 1) / 2 + (j - i);
}
// with the row offsets off[i] = packed(i, i) - i held in shared memory
__device__ __forceinline__ int packed_off(const int* off, int i, int j) {
  return i <= j ? off[i] + j : off[j] + i;
}

template <int D, int NT>
__device__ void jacobi_eigen(double* A, double* Vt, const uint32_t* blk, const int* off, double* cs, double* sn,
                             int* pp, int* qq) {
  constexpr int P = D / 2, NB = P * (P + 1) / 2;
  constexpr int BI = (NB + NT - 1) / NT, VI = P * D / NT;   // block / rotation items per thread
  static_assert(P * D % NT == 0, "V update items per thread");
  const int t = threadIdx.x;
  for (int sweep = 0; sweep < kJacobiMaxSweeps; ++sweep) {
    int rotated = 0;
    for (int r = 0; r < D - 1; ++r) {
      if (t < P) {
        // circle method: position 0 holds index 0, positions 1..D-1 rotate
        const int a = t, b = D - 1 - t;
        const int p = a == 0 ? 0 : 1 + (a - 1 + r) % (D - 1);
        const int q = 1 + (b - 1 + r) % (D - 1);
        const double app = A[off[p] + p], aqq = A[off[q] + q], apq = A[packed_off(off, p, q)];
        double c = 1.0, s = 0.0;
        if (apq != 0.0 && apq * apq > kJacobiEps * kJacobiEps * fabs(app * aqq)) {
          // tan(theta) = 2 sgn(d) a_pq / (|d| + sqrt(d^2 + 4 a_pq^2)), d = a_qq - a_pp: the smaller
          // root of t^2 + 2 tau t - 1 = 0, tau = d / (2 a_pq), without forming tau
          const double dd = aqq - app;
          const double tt = (dd >= 0.0 ? 2.0 : -2.0) * apq / (fabs(dd) + sqrt(fma(dd, dd, 4.0 * apq * apq)));
          c = rsqrt(fma(tt, tt, 1.0));
          s = tt * c;
          rotated = 1;
        }
        pp[t] = p; qq[t] = q; cs[t] = c; sn[t] = s;
      }
      __syncthreads();
#pragma unroll
      for (int u = 0; u < BI; ++u) {
        const int e = t + u * NT;
        if (e >= NB) break;
        const uint32_t kl = blk[e];
        const int k = (int)(kl >> 16), l = (int)(kl & 0xFFFFu);
        const double ck = cs[k], sk = sn[k], cl = cs[l], sl = sn[l];   // (1, 0): identity, exactly
        // d = 128: late sweeps skip most rotations, so skipping idle blocks pays; at d = 64
        // the branch-free loop is faster
        if constexpr (D == 128) {
          if (sk == 0.0 && sl == 0.0) continue;
        }
        const int pk = pp[k], qk = qq[k];
        if (k == l) {
          const int ip = off[pk] + pk, iq = off[qk] + qk, io = packed_off(off, pk, qk);
          const double aa = A[ip], ee = A[iq], bb = A[io];
          A[ip] = ck * ck * aa - 2.0 * ck * sk * bb + sk * sk * ee;
          A[iq] = sk * sk * aa + 2.0 * ck * sk * bb + ck * ck * ee;
          A[io] = sk == 0.0 ? bb : 0.0;
        } else {
          const int pl = pp[l], ql = qq[l];
          const int i00 = packed_off(off, pk, pl), i01 = packed_off(off, pk, ql);
          const int i10 = packed_off(off, qk, pl), i11 = packed_off(off, qk, ql);
          const double b00 = A[i00], b01 = A[i01], b10 = A[i10], b11 = A[i11];
          const double t00 = ck * b00 - sk * b10, t01 = ck * b01 - sk * b11;   // J_k^T B
          const double t10 = sk * b00 + ck * b10, t11 = sk * b01 + ck * b11;
          A[i00] = cl * t00 - sl * t01; A[i01] = sl * t00 + cl * t01;         // (J_k^T B) J_l
          A[i10] = cl * t10 - sl * t11; A[i11] = sl * t10 + cl * t11;
        }
      }
#pragma unroll
      for (int u = 0; u < VI; ++u) {   // V <- V J
        const int e = t + u * NT;
        const int k = e / D, i = e % D;
        const double c = cs[k], s = sn[k];
        if constexpr (D == 128) {
          if (s == 0.0) continue;
        }
        const int p = pp[k], q = qq[k];
        const double vp = Vt[p * D + i], vq = Vt[q * D + i];
        Vt[p * D + i] = c * vp - s * vq;
        Vt[q * D + i] = s * vp + c * vq;
      }
      __syncthreads();
    }
    if (!__syncthreads_or(rotated)) break;
  }
}

// One CTA per tensor-head th. M[th]: the metric whose root transforms this
// tensor (the identity without the transform); C[th]: covariance of the
// (scaled) raw rows. Writes W[th] transposed (D x D, W[th][k][j] = entry k of
// w_j, j in order of descending eigenvalue) and uses scratch[th] (2 D x D).
//
// Any factor F with F F^T = M serves in place of the symmetric root R: F = R O
// for an orthogonal O, so F^T C F = O^T (R C R) O has eigenvectors O^T u_j and
// F O^T u_j = R u_j. F comes from a pivoted Cholesky factorisation (Higham,
// "Accuracy and Stability of Numerical Algorithms", Section 10.3: pivot on the
// largest remaining diagonal entry, stop when it falls to D eps max(diag M)),
// D steps instead of a second Jacobi solve. The sign of each w_j is then set
// on w_j itself, which does not depend on the factor.
template <int D>
__global__ void __launch_bounds__(BasisCfg<D>::kThreads, 1) diag_basis_kernel(const double* __restrict__ M,
                                                                             const double* __restrict__ C,
                                                                             double* __restrict__ scratch,
                                                                             double* __restrict__ W) {
  using Cfg = BasisCfg<D>;
  constexpr int NT = Cfg::kThreads, P = Cfg::P;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* A = reinterpret_cast<double*>(smem_raw);                  // packed symmetric
  double* Vt = A + Cfg::kPacked;                                     // D x D
  uint32_t* blk = reinterpret_cast<uint32_t*>(Vt + D * D);           // pair blocks (k, l), k <= l
  __shared__ double cs[P], sn[P], lam[D], sgn[D];
  __shared__ int pp[P], qq[P], rnk[D], off[D], used[D];
  __shared__ double piv_d, piv_inv, tol_s;
  __shared__ int piv_s, stop_s;
  const int th = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const double* Mg = M + (size_t)th * D * D;
  const double* Cg = C + (size_t)th * D * D;
  double* Fg = scratch + (size_t)th * 2 * D * D;   // F transposed: Fg[k][i] = F[i][k]
  double* Tg = Fg + D * D;
  double* Wg = W + (size_t)th * D * D;

  if (t < D) { off[t] = packed<D>(t, t) - t; used[t] = 0; }
  if (t < P) {
    const int base = t * P - t * (t - 1) / 2;
    for (int l = t; l < P; ++l) blk[base + (l - t)] = ((uint32_t)t << 16) | (uint32_t)l;
  }
  if (t == 0) stop_s = 0;
  for (int e = t; e < D * D; e += NT) {
    const int i = e / D, j = e % D;
    if (j >= i) A[packed<D>(i, j)] = Mg[e];
    Vt[e] = 0.0;
  }
  __syncthreads();
  // 1. M = F F^T, F[i][k] in Vt (row-major); columns after a stop stay zero
  for (int k = 0; k < D; ++k) {
    if (warp == 0) {
      double best = -1.0;
      int bi = D;
      for (int i = lane; i < D; i += 32)
        if (!used[i]) {
          const double v = A[off[i] + i];
          if (v > best) { best = v; bi = i; }
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
      }
      if (lane == 0) {
        if (k == 0) tol_s = best * (double)D * kJacobiEps;
        if (bi >= D || !(best > tol_s)) {
          stop_s = 1;
        } else {
          const double dk = sqrt(best);
          piv_s = bi; piv_d = dk; piv_inv = 1.0 / dk; used[bi] = 1;
        }
      }
    }
    __syncthreads();
    if (stop_s) break;
    const int p = piv_s;
    const double dk = piv_d, inv = piv_inv;
    for (int i = t; i < D; i += NT)
      Vt[i * D + k] = (i == p) ? dk : (used[i] ? 0.0 : A[packed_off(off, i, p)] * inv);
    __syncthreads();
    for (int e = t; e < D * D; e += NT) {   // Schur complement on the rows not yet pivoted
      const int i = e / D, j = e % D;
      if (j >= i && !used[i] && !used[j]) A[off[i] + j] -= Vt[i * D + k] * Vt[j * D + k];
    }
    __syncthreads();
  }
  for (int e = t; e < D * D; e += NT) {
    const int i = e / D, k = e % D;
    Fg[k * D + i] = Vt[e];
  }
  // 2. C F, then the upper triangle of F^T (C F)
  for (int e = t; e < D * D; e += NT) {
    const int i = e / D, j = e % D;
    double acc = 0.0;
#pragma unroll 4
    for (int k = 0; k < D; ++k) acc = fma(Cg[i * D + k], Vt[k * D + j], acc);
    Tg[e] = acc;
  }
  __syncthreads();
  for (int e = t; e < D * D; e += NT) {
    const int i = e / D, j = e % D;
    if (j < i) continue;
    double acc = 0.0;
#pragma unroll 4
    for (int k = 0; k < D; ++k) acc = fma(Vt[k * D + i], Tg[k * D + j], acc);
    A[packed<D>(i, j)] = acc;
  }
  __syncthreads();
  for (int e = t; e < D * D; e += NT) Vt[e] = (e / D == e % D) ? 1.0 : 0.0;
  __syncthreads();
  // 3. F^T C F = U' diag(mu) U'^T
  jacobi_eigen<D, NT>(A, Vt, blk, off, cs, sn, pp, qq);
  if (t < D) lam[t] = A[off[t] + t];
  __syncthreads();
  if (t < D) {
    const double mu = lam[t];
    int r = 0;
    for (int i = 0; i < D; ++i) r += (lam[i] > mu) || (lam[i] == mu && i < t);
    rnk[t] = r;
  }
  __syncthreads();
  // 4. w_j = F u'_j into column rank(j), then each column signed by its largest-magnitude entry
  for (int e = t; e < D * D; e += NT) {
    const int j = e / D, c = e % D;
    double acc = 0.0;
#pragma unroll 4
    for (int k = 0; k < D; ++k) acc = fma(Fg[k * D + c], Vt[j * D + k], acc);
    Wg[(size_t)c * D + rnk[j]] = acc;
  }
  __syncthreads();
  if (t < D) {
    double best = -1.0, v = 0.0;
    for (int c = 0; c < D; ++c) {
      const double x = Wg[(size_t)c * D + t];
      if (fabs(x) > best) { best = fabs(x); v = x; }
    }
    sgn[t] = v < 0.0 ? -1.0 : 1.0;
  }
  __syncthreads();
  for (int e = t; e < D * D; e += NT) Wg[e] *= sgn[e % D];
}

// ---------------------------------------------------------------------------
// Per set of one level: the same sample as the basic splitting (min(d, |S|)
// members at p_j = floor((j |S| + r) / m)), its coordinates z_ij = s_i x_i . w_j
// (s_i the query scale, 1 for keys) as a 16 x 16-thread tile product in fp64,
// the variance of every coordinate over the sample (mean first, then the
// squared deviations), the coordinate of highest variance (lowest index on a
// tie), and w_j* written as the set's direction.
// ---------------------------------------------------------------------------
template <typename T, int D>
struct DiagDirCfg {
  static constexpr int kThreads = 256;
  static constexpr int TI = D / 16;     // sample rows per thread (stride 16)
  static constexpr int TJ = D / 16;     // coordinates per thread (stride 16)
  static constexpr int KC = 64;         // columns staged in fp64 at a time
  static constexpr int XS = KC + 1;     // fp64 row stride of the staged sample
  static constexpr int VEC = 16 / (int)sizeof(T);          // elements per 16-byte chunk
  static constexpr int CPR = D / VEC;                       // chunks per row
  static constexpr int NCH = D * CPR / kThreads;            // chunks per thread
  static_assert(D * CPR % kThreads == 0, "sample chunks per thread");
  static constexpr size_t kSmem = (size_t)D * D * 8 + (size_t)D * XS * 8;
};

template <typename T, int D>
__global__ void __launch_bounds__(256) diag_dir_kernel(const T* __restrict__ Q, const T* __restrict__ K,
                                                       TensorLayout TL, int n, const TreeNode* __restrict__ nodes,
                                                       int lvl_begin, int nodes_in_level, int npc,
                                                       const double* __restrict__ W,
                                                       const double* __restrict__ inv_s,
                                                       const int* __restrict__ idx, int NI,
                                                       double* __restrict__ wvec, uint64_t seed, int head_base,
                                                       int tsel) {
  using Cfg = DiagDirCfg<T, D>;
  constexpr int TI = Cfg::TI, TJ = Cfg::TJ, KC = Cfg::KC, XS = Cfg::XS;
  constexpr int VEC = Cfg::VEC, CPR = Cfg::CPR, NCH = Cfg::NCH;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* Wt = reinterpret_cast<double*>(smem_raw);                     // Wt[k][j] = w_j[k]
  double* xs = reinterpret_cast<double*>(smem_raw + (size_t)D * D * 8);  // sample rows, KC columns
  __shared__ double red[16][D];
  __shared__ double mean_s[D], ssc[D];
  __shared__ int srow[D];
  __shared__ int jbest_s;
  const int th = tsel < 0 ? (int)blockIdx.y : 2 * (int)blockIdx.y + tsel, bh = th >> 1, tensor = th & 1;
  const int t = threadIdx.x, ty = t / 16, tx = t % 16;
  const T* X = (tensor == 0 ? Q : K) + TL.head(bh);
  {
    // the basis arrives transposed: a straight 16-byte copy, all loads of a thread in flight
    const double2* src = reinterpret_cast<const double2*>(W + (size_t)th * D * D);
    double2* dst = reinterpret_cast<double2*>(Wt);
    constexpr int N2 = D * D / 2, PER = N2 / 256;
    double2 v[PER < 16 ? PER : 16];
#pragma unroll
    for (int u0 = 0; u0 < PER; u0 += 16) {
#pragma unroll
      for (int u = 0; u < 16 && u0 + u < PER; ++u) v[u] = src[(u0 + u) * 256 + t];
#pragma unroll
      for (int u = 0; u < 16 && u0 + u < PER; ++u) dst[(u0 + u) * 256 + t] = v[u];
    }
  }
  const int first = blockIdx.x * npc, last = min(nodes_in_level, first + npc);
  for (int local = first; local < last; ++local) {
    const int node_id = lvl_begin + local;
    const TreeNode nd = nodes[node_id];
    const int m = min(D, nd.size);
    const uint64_t key = node_stream(seed, (uint64_t)(head_base + bh), (uint64_t)tensor, nd.heap);
    const uint64_t r = (nd.size > m) ? (splitmix64(key ^ kSampleTag) % (uint64_t)nd.size) : 0ull;
    __syncthreads();   // the previous set is done with every shared array (and Wt is loaded)
    if (t < D) {
      int row = 0;
      double sc = 0.0;
      if (t < m) {
        const int pos = (nd.size > m) ? (int)(((uint64_t)t * (uint64_t)nd.size + r) / (uint64_t)m) : t;
        row = idx ? idx[(size_t)th * n + nd.off + pos] : nd.off + pos;
        sc = (tensor == 0) ? inv_s[(size_t)bh * n + row] : 1.0;
      }
      srow[t] = row;
      ssc[t] = sc;
    }
    __syncthreads();
    double acc[TI][TJ];
#pragma unroll
    for (int i = 0; i < TI; ++i)
#pragma unroll
      for (int j = 0; j < TJ; ++j) acc[i][j] = 0.0;
#pragma unroll
    for (int kc = 0; kc < D; kc += KC) {
      // this column block's 16-byte chunks of the sample, all of a thread's loads
      // in flight (rows >= m are zero), converted once to fp64
      if (kc > 0) __syncthreads();   // the previous column block's products are done
      constexpr int NB8 = NCH < 8 ? NCH : 8;   // chunks in flight per batch
#pragma unroll
      for (int u0 = 0; u0 < NCH; u0 += NB8) {
        uint4 raw[NB8];
#pragma unroll
        for (int u = 0; u < NB8; ++u) {
          const int e = (u0 + u) * 256 + t, j = e / CPR, k0 = (e % CPR) * VEC;
          raw[u] = make_uint4(0u, 0u, 0u, 0u);
          if (j < m && k0 >= kc && k0 < kc + KC)
            raw[u] = *reinterpret_cast<const uint4*>(X + (size_t)srow[j] * TL.sn + k0);
        }
#pragma unroll
        for (int u = 0; u < NB8; ++u) {
          const int e = (u0 + u) * 256 + t, j = e / CPR, k0 = (e % CPR) * VEC;
          if (k0 >= kc && k0 < kc + KC) {
            const T* v = reinterpret_cast<const T*>(&raw[u]);
#pragma unroll
            for (int q = 0; q < VEC; ++q) xs[j * XS + (k0 - kc) + q] = (double)to_f32(v[q]);
          }
        }
      }
      __syncthreads();
#pragma unroll 2
      for (int k = 0; k < KC; ++k) {
        double a[TI], b[TJ];
#pragma unroll
        for (int i = 0; i < TI; ++i) a[i] = xs[(ty + 16 * i) * XS + k];
#pragma unroll
        for (int j = 0; j < TJ; ++j) b[j] = Wt[(kc + k) * D + tx + 16 * j];
#pragma unroll
        for (int i = 0; i < TI; ++i)
#pragma unroll
          for (int j = 0; j < TJ; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
      }
    }
    // coordinates (rows >= m are zero and excluded); column sums
#pragma unroll
    for (int i = 0; i < TI; ++i) {
      const double sc = ssc[ty + 16 * i];
#pragma unroll
      for (int j = 0; j < TJ; ++j) acc[i][j] *= sc;
    }
#pragma unroll
    for (int j = 0; j < TJ; ++j) {
      double p = 0.0;
#pragma unroll
      for (int i = 0; i < TI; ++i)
        if (ty + 16 * i < m) p += acc[i][j];
      red[ty][tx + 16 * j] = p;
    }
    __syncthreads();
    if (t < D) {
      double sum = 0.0;
#pragma unroll
      for (int g = 0; g < 16; ++g) sum += red[g][t];
      mean_s[t] = sum / (double)m;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < TJ; ++j) {
      const double mu = mean_s[tx + 16 * j];
      double p = 0.0;
#pragma unroll
      for (int i = 0; i < TI; ++i)
        if (ty + 16 * i < m) {
          const double dv = acc[i][j] - mu;
          p = fma(dv, dv, p);
        }
      red[ty][tx + 16 * j] = p;
    }
    __syncthreads();
    if (t < 32) {
      double best = -1.0;
      int bj = D;
      for (int j = t; j < D; j += 32) {
        double v = 0.0;
#pragma unroll
        for (int g = 0; g < 16; ++g) v += red[g][j];
        if (v > best) { best = v; bj = j; }   // ascending j: the first maximum is kept
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
        if (ob > best || (ob == best && oj < bj)) { best = ob; bj = oj; }
      }
      if (t == 0) jbest_s = bj < D ? bj : 0;
    }
    __syncthreads();
    const int jb = jbest_s;
    for (int c = t; c < D; c += 256) wvec[((size_t)th * NI + node_id) * D + c] = Wt[c * D + jb];
  }
}

}  // namespace

cudaError_t launch_diag_basis(int D, int TH, int BH, int nch, int n, const double* part, const double* M,
                              double* C, double* scratch, double* W, cudaStream_t st) {
  (void)BH;
  if (D == 64) {
    cov_reduce_kernel<64><<<dim3(64 * 64 / 256, TH), 256, 0, st>>>(part, nch, n, C);
    const size_t smem = BasisCfg<64>::kSmem;
    cudaFuncSetAttribute(diag_basis_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    diag_basis_kernel<64><<<TH, BasisCfg<64>::kThreads, smem, st>>>(M, C, scratch, W);
  } else {
    cov_reduce_kernel<128><<<dim3(128 * 128 / 256, TH), 256, 0, st>>>(part, nch, n, C);
    const size_t smem = BasisCfg<128>::kSmem;
    cudaFuncSetAttribute(diag_basis_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    diag_basis_kernel<128><<<TH, BasisCfg<128>::kThreads, smem, st>>>(M, C, scratch, W);
  }
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_diag_dir(const T* Q, const T* K, TensorLayout TL, int n, const TreeNode* nodes, int lvl_begin,
                            int nodes_in_level, int TH, const double* W, const double* inv_s, const int* idx,
                            int NI, double* wvec, uint64_t seed, int head_base, int tsel, cudaStream_t st) {
  using Cfg = DiagDirCfg<T, D>;
  const int per_sm = D == 64 ? 3 : 1;   // CTAs resident per SM (shared memory)
  const int npc = (int)(((long long)nodes_in_level * TH + 148 * per_sm - 1) / (148 * per_sm));
  cudaFuncSetAttribute(diag_dir_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::kSmem);
  // TH: the grid rows (every tensor-head, or one tensor's heads when tsel >= 0)
  diag_dir_kernel<T, D><<<dim3((nodes_in_level + npc - 1) / npc, TH), Cfg::kThreads, Cfg::kSmem, st>>>(
      Q, K, TL, n, nodes, lvl_begin, nodes_in_level, npc, W, inv_s, idx, NI, wvec, seed, head_base, tsel);
  return cudaGetLastError();
}

template cudaError_t launch_diag_dir<__nv_bfloat16, 64>(const __nv_bfloat16*, const __nv_bfloat16*, TensorLayout, int,
                                                         const TreeNode*, int, int, int, const double*,
                                                         const double*, const int*, int, double*, uint64_t, int, int,
                                                         cudaStream_t);
template cudaError_t launch_diag_dir<__nv_bfloat16, 128>(const __nv_bfloat16*, const __nv_bfloat16*, TensorLayout, int,
                                                          const TreeNode*, int, int, int, const double*,
                                                          const double*, const int*, int, double*, uint64_t, int, int,
                                                          cudaStream_t);
template cudaError_t launch_diag_dir<float, 64>(const float*, const float*, TensorLayout, int, const TreeNode*, int, int,
                                                int, const double*, const double*, const int*, int, double*,
                                                uint64_t, int, int, cudaStream_t);
template cudaError_t launch_diag_dir<float, 128>(const float*, const float*, TensorLayout, int, const TreeNode*, int, int,
                                                 int, const double*, const double*, const int*, int, double*,
                                                 uint64_t, int, int, cudaStream_t);

}  // namespace ca
