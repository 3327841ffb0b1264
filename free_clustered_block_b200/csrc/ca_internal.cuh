// Internal declarations shared by the libca translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/ca.h"

namespace ca {

// ---------------------------------------------------------------------------
// Recursion tree of basic recursive splitting (PDDP).
//
// ClusterAttention paper, Section 3.1 "Overview" and Section 3.2.1: every split
// puts the multiple of c closest to |S|/2 below the threshold (the smaller
// multiple on an exact tie); splitting repeats until all sets but at most one
// hold c vectors. The shape therefore depends only on (n, c) and is planned
// before any launch. Children of a node: the lower part (t vectors) on the
// left, the rest on the right, so the one short set is always the last leaf
// and a node's first slot in the final order is also its token offset.
// ---------------------------------------------------------------------------
struct TreeNode {
  int off;      // first slot of the node in left-to-right order
  int size;     // vectors in the node
  int t;        // vectors put below the split (multiple of c)
  int parent;   // index of the parent internal node, -1 for the root
  uint64_t heap;  // heap index (root 1, children 2i, 2i+1): names the node's random stream
};

__host__ __device__ inline int split_count(int size, int c) {
  int j_lo = size / (2 * c);
  int j_hi = (size + 2 * c - 1) / (2 * c);
  long long t_lo = (long long)c * j_lo, t_hi = (long long)c * j_hi;
  long long e_lo = 2 * t_lo - size; if (e_lo < 0) e_lo = -e_lo;
  long long e_hi = 2 * t_hi - size; if (e_hi < 0) e_hi = -e_hi;
  return (int)(e_hi < e_lo ? t_hi : t_lo);
}

// Internal nodes in breadth-first order; level l holds nodes
// [level_begin[l], level_begin[l+1]). Returns the number of levels (0 when
// n <= c: the single cluster needs no split). `nodes` needs room for
// ceil(n/c) - 1 entries, `level_begin` for levels + 1 entries.
__host__ __device__ inline int plan_tree(int n, int c, TreeNode* nodes, int* level_begin,
                                         int max_levels) {
  level_begin[0] = 0;
  if (n <= c) return 0;
  nodes[0].off = 0; nodes[0].size = n; nodes[0].t = split_count(n, c);
  nodes[0].parent = -1; nodes[0].heap = 1;
  int count = 1, begin = 0, end = 1, lvl = 0;
  while (begin < end && lvl < max_levels) {
    level_begin[lvl] = begin;
    for (int i = begin; i < end; ++i) {
      TreeNode nd = nodes[i];
      int ls = nd.t, rs = nd.size - nd.t;
      if (ls > c) {
        TreeNode& ch = nodes[count++];
        ch.off = nd.off; ch.size = ls; ch.t = split_count(ls, c); ch.parent = i; ch.heap = 2 * nd.heap;
      }
      if (rs > c) {
        TreeNode& ch = nodes[count++];
        ch.off = nd.off + ls; ch.size = rs; ch.t = split_count(rs, c); ch.parent = i;
        ch.heap = 2 * nd.heap + 1;
      }
    }
    begin = end; end = count; ++lvl;
  }
  level_begin[lvl] = count;
  return lvl;
}

constexpr int kMaxLevels = 40;

// Host-side summary of the tree for launch sizing.
struct TreePlan {
  int n = 0, c = 0, C = 0, levels = 0, internal = 0;
  int level_begin[kMaxLevels + 1] = {0};
  int level_max_size[kMaxLevels] = {0};
};
bool host_plan(int n, int c, TreePlan* plan);   // false if the tree is too deep

// ---------------------------------------------------------------------------
// Counter-based generator: SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) and
// Box-Muller normals. Streams are keyed per recursion node.
// ---------------------------------------------------------------------------
__host__ __device__ inline uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__host__ __device__ inline uint64_t node_stream(uint64_t seed, uint64_t bh, uint64_t tensor,
                                                uint64_t heap) {
  uint64_t x = splitmix64(seed);
  x = splitmix64(x ^ bh);
  return splitmix64(x ^ (((tensor & 0xFFFFull) << 48) | (heap & ((1ull << 48) - 1))));
}
constexpr uint64_t kSampleTag = 0x5A3C96E10F87D2B4ull;

// Order-preserving map of a double to uint64 (after -0.0 -> +0.0).
__device__ __forceinline__ uint64_t ordered_key(double v) {
  v = v + 0.0;
  uint64_t b = (uint64_t)__double_as_longlong(v);
  return (b & 0x8000000000000000ull) ? ~b : (b | 0x8000000000000000ull);
}

// Key cluster size and the cluster counts of a (validated) shape.
inline int key_c(const ca_shape* s) { return s->c_k ? s->c_k : s->c; }

// Where the caller's Q, K, V and O keep element j of token r of head bh = b H + h:
// b sb + h sh + r sn + j (elements).
struct TensorLayout {
  long long sb, sh, sn;
  int H;
  __host__ __device__ __forceinline__ long long head(int bh) const {
    // head-major: every head one stride apart (no integer division, which
    // would use the MUFU unit that the attention's exponentials keep busy)
    if (sb == (long long)H * sh) return (long long)bh * sh;
    return (long long)(bh / H) * sb + (long long)(bh % H) * sh;
  }
};
inline TensorLayout tensor_layout(const ca_shape* s) {
  TensorLayout L;
  const long long d = s->d, N = s->N_alloc;
  L.H = s->H;
  if (s->layout == CA_LAYOUT_BNHD) {
    const long long Ht = s->H_total > 0 ? s->H_total : s->H;
    L.sn = Ht * d; L.sh = d; L.sb = N * Ht * d;
  } else {
    L.sn = d; L.sh = N * d; L.sb = (long long)s->H * N * d;
  }
  return L;
}
inline bool layout_contiguous(const ca_shape* s) {
  return s->layout == CA_LAYOUT_BHND || s->H_total == 0 || s->H_total == s->H;
}
inline int num_q_clusters(const ca_shape* s) { return (s->n_valid + s->c - 1) / s->c; }
inline int num_k_clusters(const ca_shape* s) { return (s->n_valid + key_c(s) - 1) / key_c(s); }

// ---------------------------------------------------------------------------
// Workspace layouts (byte offsets; every region 256-byte aligned).
// ---------------------------------------------------------------------------
inline size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }

struct ClusterWs {
  size_t nodes, level_begin, nodes_k, level_begin_k, M, kmean, colsum_part, met_part, inv_s, idx0, idx1, keys,
      zvec, wvec, sel, chunk_cnt, cov, basis, basis_scratch, total;
  int nch = 0;       // metric row chunks
  int pch_max = 0;   // partition chunks per node, max over levels
  int TH = 0, BH = 0;
  int NI = 0;        // internal nodes per tensor-head, the larger of the two trees
};
constexpr int kMetricChunk = 2048;     // rows per metric partial
constexpr int kPartChunk = 2048;       // positions per partition chunk
// plan_k: the key tree when the key cluster size differs (else plan again)
bool cluster_ws_layout(const ca_shape* s, const TreePlan& plan, const TreePlan& plan_k, ClusterWs* ws);

// Diagonalized splitting (diag.cu): covariances from the Gram partials, the
// principal-component directions W per tensor-head, and the per-level choice
// of the highest-variance coordinate.
cudaError_t launch_diag_basis(int D, int TH, int BH, int nch, int n, const double* part, const double* M,
                              double* C, double* scratch, double* W, cudaStream_t st);
template <typename T, int D>
cudaError_t launch_diag_dir(const T* Q, const T* K, TensorLayout TL, int n, const TreeNode* nodes, int lvl_begin,
                            int nodes_in_level, int TH, const double* W, const double* inv_s, const int* idx,
                            int NI, double* wvec, uint64_t seed, int head_base, int tsel, cudaStream_t st);

struct AttendWs {
  size_t qp, kp, vp, kbar_hl, vbar_hl, vbar32, kbar32, logcnt, total;
  int C = 0;      // query clusters
  int Ck = 0;     // key clusters
  int Cpad = 0;   // key clusters rounded up to 128 (compensation tiles)
};
bool attend_ws_layout(const ca_shape* s, AttendWs* ws);

// ---------------------------------------------------------------------------
// Device error word and bounded waits.
// ---------------------------------------------------------------------------
// The error word lives in attend_tc.cu; other units reach it through these.
uint64_t wait_limit();                            // time limit (ns) of bounded waits
cudaError_t device_error_read_clear(unsigned* out, cudaStream_t st);
cudaError_t launch_bounded_wait_check(uint64_t limit_ns, int arrive, cudaStream_t st);
cudaError_t launch_exp2_poly_check(const float* x, float* y, int n, cudaStream_t st);
void set_wait_limit(uint64_t limit_ns);

// ---------------------------------------------------------------------------
// Launchers (each returns cudaGetLastError() of its launches).
// ---------------------------------------------------------------------------
cudaError_t launch_cluster(const void* Q, const void* K, const ca_shape* s,
                           const ca_cluster_params* p, const ca_clusters* out,
                           const TreePlan& plan, const TreePlan& plan_k, const ClusterWs& L, char* ws,
                           cudaStream_t st);
cudaError_t launch_route(const ca_shape* s, int Cq, int Ck, const double* qbar, const double* kbar, int k,
                         int32_t* kept_idx, uint32_t* kept_bits, int32_t* kept_count, cudaStream_t st);
size_t route_adaptive_smem(int C);
cudaError_t launch_route_adaptive(const ca_shape* s, int Cq, int Ck, const double* qbar, const double* kbar,
                                  const int32_t* count_k, double recall, int min_count, int k, int32_t* kept_idx,
                                  uint32_t* kept_bits, int32_t* kept_count, cudaStream_t st);
cudaError_t launch_attend_prep(const void* Q, const void* K, const void* V, const ca_shape* s,
                               const ca_clusters* cl, const AttendWs& L, char* ws, cudaStream_t st);
cudaError_t launch_attend_simt(const void* Q, const void* K, const void* V, const ca_shape* s,
                               const ca_clusters* cl, const ca_routes* rt, int compensate,
                               void* O, const AttendWs& L, char* ws, cudaStream_t st);
cudaError_t launch_attend_tc(const ca_shape* s, const ca_clusters* cl, const ca_routes* rt,
                             int compensate, void* O, const AttendWs& L, char* ws, cudaStream_t st);
cudaError_t launch_dense_simt(const void* Q, const void* K, const void* V, const ca_shape* s,
                              void* O, cudaStream_t st);
cudaError_t launch_dense_tc(const void* Q, const void* K, const void* V, const ca_shape* s,
                            void* O, cudaStream_t st);
cudaError_t launch_zero_pad_rows(void* O, const ca_shape* s, cudaStream_t st);

}  // namespace ca
