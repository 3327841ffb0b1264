// Block-sparse attention with striped mean-compensation on the sm_100a
// tensor cores (tcgen05, TMEM accumulators, TMA tiles).
//
// ClusterAttention paper, Section 3.1 (attention over the kept key clusters
// of each query cluster, blocks of the permuted tokens) and Appendix A,
// eq. 21-22 (every excluded key cluster b enters the softmax with logit
// q . kbar_b / sqrt(d) + ln|b| and value vbar_b). The dense form (eq. 1) is
// the same kernel with every key block kept and no compensation.
//
// One CTA holds an SM and works on TWO 128-row query tiles at once, so the
// tensor core computes one tile's products while the other tile's softmax
// runs (512 TMEM columns: S_0, S_1 of 128 columns, O_0, O_1 of d columns):
//   warps 0-3   softmax of tile 0, one thread per query row: read the row of
//               S_j from TMEM into registers, mask / bias it, take the row
//               maximum, write P_j = 2^(S_j - m) as bf16 over the front of
//               S_j, keep the row sum; rescale the row of O only when the
//               running maximum grows by more than 2^8; finally O / l to the
//               query's original row;
//   warps 4-7   the same for tile 1;
//   warp 8      TMA producer (one thread): both Q tiles once, then a ring of
//               K slots and a ring of V slots, each slot one 128-row tile,
//               filled in a fixed order (V two entries behind K);
//   warps 9, 10 MMA issuers, one per tile (one leader lane issues each group
//               of products from precomputed descriptors): S_t = Q_t K_j^T
//               and O_t += P_t V_j in the tile's own order. At d = 128, S_t
//               of block j+1 overwrites P_t of block j, so it waits for
//               O_t += P_t V_j; at d = 64, P_t has its own TMEM columns and
//               S_t of block j+1 is computed while block j's softmax runs;
//   warp 11     idle.
// Every wait is an mbarrier try_wait, which suspends the warp until the
// phase completes: the producer and the issuers take no issue slots from the
// softmax warps that share their SM sub-partitions.
// A key block is 128 key slots: one or half of a kept key cluster (c = 128,
// 256), two kept clusters of 64 (c = 64), or 128 consecutive keys (dense).
// A compensation block is 64 key-cluster centroids: bf16 hi parts in rows
// 0-63 of the slot and lo parts in rows 64-127, so that two N = 64 products
// carry the fp64 centroid (~16 significant bits) into the fp32 accumulator.
// When both tiles of a CTA attend the same key blocks (the two halves of a
// 256-query cluster, or dense attention) each K and V tile is loaded once
// and serves both.
// Every wait is bounded: on a timeout the CTA sets the library's device error
// word (CA_ERR_TIMEOUT), drains what it issued, frees TMEM and returns.
#include <cuda.h>

#include <atomic>

#include "ca_internal.cuh"

namespace ca {

// One word per device, shared by every stream and caller of the library.
__device__ unsigned int g_device_error = 0;
// Bounded waits are timed with the global nanosecond timer.
constexpr uint64_t kDefaultWaitLimitNs = 1000000000ull;   // 1 s
static std::atomic<uint64_t> g_wait_limit_ns{0};
// Drains (letting copies and MMAs already issued finish before the CTA
// leaves) use their own bound, independent of the adjustable wait limit.
constexpr uint64_t kDrainLimitNs = 1000000000ull;

uint64_t wait_limit() {
  const uint64_t v = g_wait_limit_ns.load(std::memory_order_relaxed);
  return v ? v : kDefaultWaitLimitNs;
}
void set_wait_limit(uint64_t limit_ns) { g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed); }

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

namespace {

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t su32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void tma_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          su32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(su32(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z,
                                       int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(su32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(su32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// tcgen05.mma (A and B from shared memory, or A from TMEM) and commit, issued
// by the calling thread alone: the MMA warp's leader lane issues whole groups
// of products this way, with no per-product election.
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(b))
               : "memory");
}
__device__ __forceinline__ bool elect_one() {
  uint32_t e;
  asm volatile("{\n .reg .pred p;\n elect.sync _|p, 0xffffffff;\n selp.u32 %0, 1, 0, p;\n}\n" : "=r"(e));
  return e != 0;
}
// Commit issued by one elected lane of a converged warp.
__device__ __forceinline__ void tc_commit_elect(uint64_t* b) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(su32(b))
      : "memory");
}

#define CA_TMEM_LD32(taddr, r)                                                                              \
  asm volatile(                                                                                             \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17," \
      "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                                    \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),      \
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),            \
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),          \
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),          \
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])                                                               \
      : "r"(taddr))

#define CA_TMEM_ST32(taddr, r)                                                                              \
  asm volatile(                                                                                             \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16," \
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),                     \
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),     \
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),         \
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),        \
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])                     \
      : "memory")

#define CA_TMEM_ST16(taddr, r)                                                                              \
  asm volatile(                                                                                             \
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" \
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),  \
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])           \
      : "memory")

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// packed pairs of f32 (sm_100 f32x2 arithmetic) and the three-input max
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// 2^t0, 2^t1 on the FMA pipe, to take part of the load off the MUFU ex2
// unit. t = n + f with n = round(t): adding 1.5 * 2^23 leaves the rounded
// integer in the low mantissa bits of y, and subtracting it back gives n
// exactly, so f = t - n lies in [-1/2, 1/2]. 2^f is the cubic of least
// maximum relative error on that interval, found by the Remez exchange
// algorithm (exp2_poly_fit.py beside this file; 7.5e-5 relative). n enters
// the exponent field with one integer multiply-add (y's low bits times 2^23).
// t is clamped at -126 first: 2^-126 is as good as 0 for a bf16 P.
__device__ __forceinline__ void exp2_poly2(float t0, float t1, float& r0, float& r1) {
  constexpr float kRound = 12582912.f;   // 1.5 * 2^23
  constexpr float c0 = 9.9992805719e-01f, c1 = 6.9326096773e-01f, c2 = 2.4261112511e-01f,
                  c3 = 5.5171668530e-02f;
  const uint64_t t2 = f2_pack(fmaxf(t0, -126.f), fmaxf(t1, -126.f));
  const uint64_t y2 = add2(t2, f2_pack(kRound, kRound));
  const uint64_t n2 = add2(y2, f2_pack(-kRound, -kRound));
  const uint64_t f2 = fma2(n2, f2_pack(-1.f, -1.f), t2);
  uint64_t q2 = fma2(f2_pack(c3, c3), f2, f2_pack(c2, c2));
  q2 = fma2(q2, f2, f2_pack(c1, c1));
  q2 = fma2(q2, f2, f2_pack(c0, c0));
  float y0, y1, q0, q1;
  f2_unpack(y2, y0, y1);
  f2_unpack(q2, q0, q1);
  r0 = __int_as_float(__float_as_int(y0) * 8388608 + __float_as_int(q0));
  r1 = __int_as_float(__float_as_int(y1) * 8388608 + __float_as_int(q1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Shared-memory matrix descriptor, 128-byte swizzle (canonical layouts of the
// tcgen05 matrix descriptor: start >> 4 in bits 0-13, leading byte offset >> 4
// in 16-29, stride byte offset >> 4 in 32-45, descriptor version 1 in 46-47,
// swizzle mode 2 (128B) in 61-63).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B, A K-major,
// B K-major (b_mn = 0) or MN-major (b_mn = 1), N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void raise_timeout(volatile int* abort_flag) {
  atomicCAS(&g_device_error, 0u, (unsigned)CA_ERR_TIMEOUT);
  *abort_flag = 1;
}
// Bounded wait (limit in ns); false on timeout or when another role aborted.
// Every helper here is inlined: ptxas cannot allocate the registers of the
// kernel's setmaxnreg regions when they contain a call.
__device__ __forceinline__ bool wait_bar_slow(uint64_t* b, uint32_t parity, uint64_t limit_ns,
                                           volatile int* abort_flag) {
  const uint64_t t0 = now_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try(b, parity)) return true;
    if ((i & 31) == 0) {
      if (*abort_flag) return false;
      if (now_ns() - t0 > limit_ns) { raise_timeout(abort_flag); return false; }
    }
  }
}
// A barrier that has already flipped is taken on the first probe.
__device__ __forceinline__ bool wait_bar(uint64_t* b, uint32_t parity, uint64_t limit_ns, volatile int* abort_flag) {
  if (mbar_try(b, parity)) return true;
  return wait_bar_slow(b, parity, limit_ns, abort_flag);
}
// Bounded wait used while draining: ignores the abort flag, fixed limit.
__device__ __forceinline__ void drain_bar(uint64_t* b, uint32_t parity) {
  const uint64_t t0 = now_ns();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try(b, parity)) return;
    if ((i & 31) == 31 && now_ns() - t0 > kDrainLimitNs) return;
  }
}

// ---------------------------------------------------------------------------
// Kernel parameters and per-tile bookkeeping
// ---------------------------------------------------------------------------
struct TcParams {
  int C, c;                   // query clusters and their size
  int Ck, ck;                 // key clusters and their size
  int k, Cpad, n_valid, N_alloc;
  int tiles_per_cluster;      // c / 128 (1 when c = 64)
  int rows_per_tile;          // min(c, 128): query rows of a tile that belong to its cluster
  int n_tiles;                // sparse: query tiles over all heads
  int pair;                   // 1: a tile holds two query clusters of 64 (rows 0-63 and 64-127)
                              // and runs over the union of their kept key clusters
  int compensate;
  int J_cent;                 // compensation blocks per tile: ceil(C / 64) with compensation, else 0
  int dense;                  // 1: identity order, every key block kept
  int dense_tiles;            // dense: query tiles per head
  int dense_key_blocks;       // dense: ceil(n_valid / 128)
  float scale_log2;           // log2(e) / sqrt(d)
  const int32_t* perm_q;      // [BH][C*c]
  const int32_t* count_k;     // [BH][C]
  const int32_t* kept_idx;    // [BH][C][k]
  const int32_t* kept_count;  // [BH][C] kept per query cluster, or null (k each)
  const uint32_t* kept_bits;  // [BH][C][W]
  const float* logcnt;        // [BH][Cpad] natural log of counts (-inf past C)
  __nv_bfloat16* O;           // the caller's layout (TL)
  TensorLayout TL;            // of Q, K, V and O
  int dense_tok_inner;        // dense maps: 1 when the token dimension precedes the head dimension
  uint64_t wait_limit;
};

struct Tile {
  int exists;    // the CTA has this tile (the last CTA may have one only)
  int bh, a, sub;
  int two;       // pair mode: the tile holds query clusters a and a + 1
  int kq;        // kept key clusters
  int J_kept;    // kept key blocks
  int J;         // all blocks (kept, then compensation); 0 for a missing tile
  int qrow;      // first Q row of the tile (permuted rows; head rows in dense mode)
};

// kq_union: in pair mode, the size of the tile's union of kept clusters
// (computed by the kernel's prologue), ignored otherwise.
__device__ __forceinline__ Tile make_tile(const TcParams& p, int t, int kq_union = 0) {
  Tile T;
  T.exists = 0; T.bh = 0; T.a = 0; T.sub = 0; T.two = 0; T.kq = 0; T.J_kept = 0; T.J = 0; T.qrow = 0;
  if (p.dense) {
    const int ti = blockIdx.x * 2 + t;
    T.bh = blockIdx.y;
    if (ti < p.dense_tiles) {
      T.exists = 1;
      T.qrow = ti * 128;
      T.J_kept = p.dense_key_blocks;
      T.J = T.J_kept;
    }
    return T;
  }
  const int ti = blockIdx.x * 2 + t;
  if (ti >= p.n_tiles) return T;
  T.exists = 1;
  if (p.pair) {
    const int pairs = (p.C + 1) / 2;
    T.bh = ti / pairs;
    T.a = 2 * (ti % pairs);
    T.two = T.a + 1 < p.C;
    T.kq = kq_union;
    T.J_kept = p.ck >= 128 ? T.kq * (p.ck / 128) : (T.kq + 1) / 2;
    T.J = T.J_kept + p.J_cent;
    T.qrow = (T.bh * p.C + T.a) * p.c;
    return T;
  }
  const int per_head = p.C * p.tiles_per_cluster;
  T.bh = ti / per_head;
  const int rem = ti % per_head;
  T.a = rem / p.tiles_per_cluster;
  T.sub = rem % p.tiles_per_cluster;
  T.kq = p.kept_count ? min(max(p.kept_count[(size_t)T.bh * p.C + T.a], 0), p.k) : p.k;
  T.J_kept = p.ck >= 128 ? T.kq * (p.ck / 128) : (T.kq + 1) / 2;
  T.J = T.J_kept + p.J_cent;
  T.qrow = (T.bh * p.C + T.a) * p.c + T.sub * 128;
  return T;
}

// Position of item i of the interleaved (tile, block) order: (0,0), (1,0),
// (0,1), (1,1), ... while both tiles have blocks, then the longer tile's rest.
__device__ __forceinline__ void item_at(int i, int J0, int J1, int& t, int& j) {
  const int m = J0 < J1 ? J0 : J1;
  if (i < 2 * m) { t = i & 1; j = i >> 1; }
  else { t = J0 > J1 ? 0 : 1; j = m + (i - 2 * m); }
}

template <int D>
struct TcCfg {
  static constexpr int kSub = D / 64;                  // 64-column (128-byte) sub-tiles per row
  static constexpr int kTileBytes = 128 * D * 2;       // a Q tile, or one ring slot (128 rows)
  static constexpr int kSubBytes = 128 * 128;          // one sub-tile of a 128-row tile
  static constexpr int kKS = D == 64 ? 5 : 2;          // K ring slots
  static constexpr int kVS = D == 64 ? 5 : 2;          // V ring slots
  static constexpr int kMaxKept = 512;                 // kept list staged in shared memory
  static constexpr int kKOff = 2 * kTileBytes;
  static constexpr int kVOff = kKOff + kKS * kTileBytes;
  static constexpr int kBarOff = kVOff + kVS * kTileBytes;
  static constexpr int kBiasOff = kBarOff + 512;       // per softmax warp: 64 compensation biases
  static constexpr int kKeptOff = kBiasOff + 8 * 64 * 4;
  static constexpr int kSmem = kKeptOff + 2 * 2 * kMaxKept * 4 + 1024;   // + alignment slack
  static constexpr int kThreads = 384;
  // Registers per thread: the launch gives every thread kRegLaunch (the most
  // 384 threads can hold); then the producer / MMA warpgroup gives registers
  // back (setmaxnreg.dec) and the two softmax warpgroups take them
  // (setmaxnreg.inc), which holds one row of S in registers. The shares must
  // add up to exactly the launch's total, or the increase would wait forever;
  // the host refuses to launch a build whose register count is not kRegLaunch.
  static constexpr int kRegLaunch = 168;
  static constexpr int kRegSoftmax = 208;
  static constexpr int kRegOther = 88;
  static constexpr uint32_t kTmemCols = 512;
  // TMEM: S_t at t * 128. At d = 64, P_t has its own 64 columns (so S_t of
  // the next block can be computed while P_t is still being read) and O_t
  // follows; at d = 128 the O accumulators need the room, so P_t is written
  // over the front of S_t and S_t of the next block waits for O_t += P_t V.
  static constexpr bool kAliasP = D == 128;
  static constexpr uint32_t kPCol = kAliasP ? 0 : 256;       // P_t at kPCol + t * kPStride
  static constexpr uint32_t kPStride = kAliasP ? 128 : 64;
  static constexpr uint32_t kOCol = kAliasP ? 256 : 384;     // O_t at kOCol + t * D
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(kOCol + 2 * D <= kTmemCols, "TMEM");
  static_assert(kAliasP || kPCol + 2 * 64 <= kOCol, "TMEM: P columns");
  static_assert(kRegLaunch * kThreads == 65536 / (kThreads * 8) * 8 * kThreads, "launch register count");
  static_assert(256 * kRegSoftmax + 128 * kRegOther == kThreads * kRegLaunch, "register split");
};

// Pairs of P columns (bit q % 8 of the mask) whose exponentials run on the
// FMA pipe (exp2_poly2) instead of the MUFU unit. Measured on B200 (the
// attention of the N = 65,536 d = 64 layer): with three pairs in eight on the
// FMA pipe the kernel took 2.05 ms, with none 1.94 ms, so at d = 64 all
// exponentials stay on the MUFU unit; at d = 128 one pair in eight moves.
#ifndef CA_TC_POLY64
#define CA_TC_POLY64 0x00
#endif
#ifndef CA_TC_POLY128
#define CA_TC_POLY128 0x01
#endif

// One block of one row, from the NC values of S already in registers: mask
// or bias them, update the running maximum (lazily), and turn them into
// P = 2^(S - m) as bf16 pairs (pk) plus the row sum. Returns whether the
// maximum moved (O must then be scaled by `factor`).
template <int NC, unsigned kPoly>
__device__ __forceinline__ bool softmax_block(float (&v)[NC], uint32_t (&pk)[NC / 2], float sc, const float* bias,
                                              int v0, int v1, float& m_ref, float& l, float& factor) {
  const bool special = bias != nullptr || v0 < 64 || (NC > 64 && v1 < 64);
  if (special) {
    if (bias) {
#pragma unroll
      for (int q = 0; q < NC; ++q) v[q] = fmaf(v[q], sc, bias[q]);
    } else {
#pragma unroll
      for (int q = 0; q < NC; ++q) v[q] = ((q < 64) ? (q < v0) : (q - 64 < v1)) ? v[q] * sc : -INFINITY;
    }
  }
  float m4[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) m4[q] = -INFINITY;
#pragma unroll
  for (int q = 0; q < NC; q += 2) m4[(q >> 1) & 3] = max3(m4[(q >> 1) & 3], v[q], v[q + 1]);
  float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
  if (!special) mx *= sc;   // log2 units (masked / biased values already are)
  const bool need = mx > m_ref + 8.f;
  factor = 1.f;
  if (need) {
    factor = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - mx);
    m_ref = mx;
    l *= factor;
  }
  const float nb = (m_ref == -INFINITY) ? 0.f : -m_ref;
  const float xs = special ? 1.f : sc;
  const uint64_t xs2 = f2_pack(xs, xs), nb2 = f2_pack(nb, nb);
  uint64_t ls2[2] = {0ull, 0ull};
#pragma unroll
  for (int q = 0; q < NC / 2; ++q) {
    float t0, t1, p0, p1;
    f2_unpack(fma2(f2_pack(v[2 * q], v[2 * q + 1]), xs2, nb2), t0, t1);
    if ((kPoly >> (q & 7)) & 1u) exp2_poly2(t0, t1, p0, p1);
    else { p0 = ex2(t0); p1 = ex2(t1); }
    ls2[q & 1] = add2(ls2[q & 1], f2_pack(p0, p1));
    pk[q] = pack_bf16(p0, p1);
  }
  float a0, a1;
  f2_unpack(add2(ls2[0], ls2[1]), a0, a1);
  l += a0 + a1;
  return need;
}

template <int D>
__global__ void __launch_bounds__(TcCfg<D>::kThreads, 1)
tc_attend_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kc,
                 const __grid_constant__ CUtensorMap tm_vc, const TcParams p) {
  using Cfg = TcCfg<D>;
  constexpr int KS = Cfg::kKS, VS = Cfg::kVS;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  unsigned char* sQ = smem;                        // [2] Q tiles
  unsigned char* sK = smem + Cfg::kKOff;           // [KS] K slots
  unsigned char* sV = smem + Cfg::kVOff;           // [VS] V slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* q_full = bars;                 // [2]
  uint64_t* kfull = q_full + 2;            // [KS]
  uint64_t* kempty = kfull + KS;           // [KS]
  uint64_t* vfull = kempty + KS;           // [VS]
  uint64_t* vempty = vfull + VS;           // [VS]
  uint64_t* s_full = vempty + VS;          // [2] S_t computed
  uint64_t* s_free = s_full + 2;           // [2] S_t read into registers (128 arrivals; separate P only)
  uint64_t* p_full = s_free + 2;           // [2] P_t written (128 arrivals)
  uint64_t* pv_done = p_full + 2;          // [2] O_t += P_t V completed
  uint64_t* drain = pv_done + 2;           // [2] one per MMA issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* bias_w = reinterpret_cast<float*>(smem + Cfg::kBiasOff);   // [8 warps][64]
  int32_t* kept_s = reinterpret_cast<int32_t*>(smem + Cfg::kKeptOff);   // [2][kMaxKept]
  int32_t* kcnt_s = kept_s + 2 * Cfg::kMaxKept;                         // [2][kMaxKept]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int kq_union[2];
  if (p.pair) {
    // Pair mode: each tile runs over the union of its two query clusters'
    // kept key clusters, listed in ascending order from the OR of their
    // bitmasks; an entry's count carries which of the two keep it (bit 16:
    // the first cluster, bit 17: the second).
    int* wcnt = reinterpret_cast<int*>(bias_w);   // [2][256] word counts, free until the softmax stages biases
    const int W = (p.Ck + 31) / 32;
    for (int t = 0; t < 2; ++t) {
      const Tile B = make_tile(p, t);
      const uint32_t* r0 = p.kept_bits + ((size_t)B.bh * p.C + B.a) * W;
      const uint32_t* r1 = B.two ? r0 + W : nullptr;
      for (int w = threadIdx.x; w < W; w += Cfg::kThreads)
        wcnt[t * 256 + w] = B.exists ? __popc(r0[w] | (r1 ? r1[w] : 0u)) : 0;
    }
    __syncthreads();
    if (warp < 2) {
      // exclusive scan of the W word counts of tile `warp` (W <= 256: 8 per lane)
      const int t = warp;
      int v[8], tot = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) { const int w = lane * 8 + q; v[q] = w < W ? wcnt[t * 256 + w] : 0; tot += v[q]; }
      int inc = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      int run = inc - tot;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int w = lane * 8 + q;
        if (w < W) wcnt[t * 256 + w] = run;
        run += v[q];
      }
      if (lane == 31) kq_union[t] = inc;
    }
    __syncthreads();
    for (int t = 0; t < 2; ++t) {
      const Tile B = make_tile(p, t);
      if (!B.exists) continue;
      const uint32_t* r0 = p.kept_bits + ((size_t)B.bh * p.C + B.a) * W;
      const uint32_t* r1 = B.two ? r0 + W : nullptr;
      for (int w = threadIdx.x; w < W; w += Cfg::kThreads) {
        const uint32_t m0 = r0[w], m1 = r1 ? r1[w] : 0u;
        uint32_t u = m0 | m1;
        int o = wcnt[t * 256 + w];
        while (u) {
          const int bit = __ffs(u) - 1;
          const int b = w * 32 + bit;
          kept_s[t * Cfg::kMaxKept + o] = b;
          kcnt_s[t * Cfg::kMaxKept + o] = p.count_k[(size_t)B.bh * p.Ck + b] | (int)(((m0 >> bit) & 1u) << 16) |
                                          (int)(((m1 >> bit) & 1u) << 17);
          ++o;
          u &= u - 1;
        }
      }
    }
    __syncthreads();
  }
  const Tile T0 = make_tile(p, 0, p.pair ? kq_union[0] : 0), T1 = make_tile(p, 1, p.pair ? kq_union[1] : 0);
  // both tiles attend the same key blocks: dense attention, or the two
  // halves of one 256-query cluster
  const bool shared_kv = T1.J > 0 && (p.dense || (p.c == 256 && T0.bh == T1.bh && T0.a == T1.a));
  // kept lists (and the kept clusters' sizes) in shared memory when they fit
  // (pair mode: already there, the unions)
  const bool kept_sm0 = !p.dense && (p.pair || T0.kq <= Cfg::kMaxKept);
  const bool kept_sm1 = !p.dense && (p.pair || T1.kq <= Cfg::kMaxKept);
  const int32_t* kept_g0 = p.dense ? nullptr : p.kept_idx + ((size_t)T0.bh * p.C + T0.a) * p.k;
  const int32_t* kept_g1 = p.dense ? nullptr : p.kept_idx + ((size_t)T1.bh * p.C + T1.a) * p.k;
  if (!p.pair && kept_sm0 && T0.J > 0) {
    for (int i = threadIdx.x; i < T0.kq; i += Cfg::kThreads) {
      const int b = kept_g0[i];
      kept_s[i] = b;
      kcnt_s[i] = p.count_k[(size_t)T0.bh * p.Ck + b];
    }
  }
  if (!p.pair && kept_sm1 && T1.J > 0) {
    for (int i = threadIdx.x; i < T1.kq; i += Cfg::kThreads) {
      const int b = kept_g1[i];
      kept_s[Cfg::kMaxKept + i] = b;
      kcnt_s[Cfg::kMaxKept + i] = p.count_k[(size_t)T1.bh * p.Ck + b];
    }
  }
  // dense mode: tile of 128 tokens of head bh from a 4-D map over (d, tokens,
  // heads, batch) or (d, heads, tokens, batch), whichever orders the strides
  // (head and batch of each tile computed once: no division per load)
  auto tma_dense = [&](void* dst, const CUtensorMap* map, uint64_t* bar, int x, int row, int hd, int bt) {
    if (p.dense_tok_inner) tma_4d(dst, map, bar, x, row, hd, bt);
    else tma_4d(dst, map, bar, x, hd, row, bt);
  };
  auto kept_at = [&](int t, int i) -> int {
    const bool sm = t ? kept_sm1 : kept_sm0;
    return sm ? kept_s[t * Cfg::kMaxKept + i] : (t ? kept_g1 : kept_g0)[i];
  };

  if (threadIdx.x == 0) {
    // with shared K/V tiles a slot is free once both tiles' products read it
    const uint32_t users = shared_kv ? 2u : 1u;
    for (int s = 0; s < KS; ++s) { mbar_init(&kfull[s], 1); mbar_init(&kempty[s], users); }
    for (int s = 0; s < VS; ++s) { mbar_init(&vfull[s], 1); mbar_init(&vempty[s], users); }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&q_full[t], 1);
      mbar_init(&s_full[t], 1);
      mbar_init(&s_free[t], 128);
      mbar_init(&p_full[t], 128);
      mbar_init(&pv_done[t], 1);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                 "r"(Cfg::kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t limit = p.wait_limit;
  const int NI = T0.J + T1.J;                   // (tile, block) items
  const int NR = shared_kv ? T0.J : NI;         // ring items (one per item, or one per block when shared)
  // Ring index of block j of tile t: the producer fills the rings in the
  // interleaved order (0,0), (1,0), (0,1), (1,1), ... (or one entry per block
  // when the tiles share K/V); each tile consumes its own entries in order.
  const int m01 = T0.J < T1.J ? T0.J : T1.J;
  auto ring_of = [&](int t, int j) -> int {
    if (shared_kv) return j;
    return j < m01 ? 2 * j + t : 2 * m01 + (j - m01);
  };

  if (warp >= 8) {
   // producer / MMA warpgroup: gives registers to the softmax warpgroups
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(Cfg::kRegOther));
   if (warp == 8) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      bool ok = true;
      // dense mode: both tiles are of head T0.bh (head and batch computed once)
      const int dh = T0.bh % p.TL.H, db = T0.bh / p.TL.H;
      for (int t = 0; t < 2; ++t) {
        const Tile& Tt = t ? T1 : T0;
        if (Tt.J == 0) continue;
        mbar_expect_tx(&q_full[t], Cfg::kTileBytes);
        for (int sb = 0; sb < Cfg::kSub; ++sb) {
          unsigned char* dst = sQ + t * Cfg::kTileBytes + sb * Cfg::kSubBytes;
          if (p.dense) tma_dense(dst, &tm_q, &q_full[t], sb * 64, Tt.qrow, dh, db);
          else tma_2d(dst, &tm_q, &q_full[t], sb * 64, Tt.qrow);
        }
      }
      // Load the K (is_v = 0) or V tile of ring item r into `dst`.
      auto load_item = [&](int r, bool is_v, unsigned char* dst, uint64_t* bar) {
        int t = 0, j = r;
        if (!shared_kv) item_at(r, T0.J, T1.J, t, j);
        const Tile& Tt = t ? T1 : T0;
        mbar_expect_tx(bar, Cfg::kTileBytes);
        const CUtensorMap* mk = is_v ? &tm_v : &tm_k;
        const CUtensorMap* mc = is_v ? &tm_vc : &tm_kc;
        for (int sb = 0; sb < Cfg::kSub; ++sb) {
          unsigned char* d = dst + sb * Cfg::kSubBytes;
          if (p.dense) {
            tma_dense(d, mk, bar, sb * 64, j * 128, dh, db);
          } else if (j < Tt.J_kept) {
            if (p.ck >= 128) {
              // c_k is 128 or 256: one or two key blocks per kept cluster (a
              // shift, not a division: this thread shares its SM sub-partition's
              // MUFU unit with a softmax warp's exponentials)
              const int sh = p.ck >> 8;
              tma_2d(d, mk, bar, sb * 64, (Tt.bh * p.Ck + kept_at(t, j >> sh)) * p.ck + (j & sh) * 128);
            } else {
              // two key clusters of 64; an odd count repeats the first (its
              // columns are masked, and its values stay finite)
              const int b0 = kept_at(t, 2 * j);
              const int b1 = (2 * j + 1 < Tt.kq) ? kept_at(t, 2 * j + 1) : b0;
              tma_2d(d, mk, bar, sb * 64, (Tt.bh * p.Ck + b0) * 64);
              tma_2d(d + 64 * 128, mk, bar, sb * 64, (Tt.bh * p.Ck + b1) * 64);
            }
          } else {
            const int cb = j - Tt.J_kept;
            tma_2d(d, mc, bar, sb * 64, (Tt.bh * (p.Cpad / 64) + cb) * 128);
          }
        }
      };
      // Fixed order: K of ring entry i, then V of entry i - kVLag (V is
      // consumed a softmax later than K). Each slot is refilled once the
      // products that read it have completed; the waits are bounded
      // try_waits, so the warp sleeps in hardware meanwhile.
      constexpr int kVLag = 2;
      int kn = 0, vn = 0;   // entries whose K / V copies were issued
      while (ok && vn < NR) {
        if (kn < NR) {
          if (!(ok = wait_bar(&kempty[kn % KS], ((kn / KS) & 1) ^ 1, limit, abort_flag))) break;
          load_item(kn, false, sK + (kn % KS) * Cfg::kTileBytes, &kfull[kn % KS]);
          ++kn;
        }
        // V of the entries up to kn - kVLag, or of all the rest once every K is issued
        const int vlim = kn < NR ? kn - kVLag : NR;
        while (vn < vlim) {
          if (!(ok = wait_bar(&vempty[vn % VS], ((vn / VS) & 1) ^ 1, limit, abort_flag))) break;
          load_item(vn, true, sV + (vn % VS) * Cfg::kTileBytes, &vfull[vn % VS]);
          ++vn;
        }
      }
      if (!ok) {
        // Let every copy already issued land before the CTA leaves.
        if (T0.J > 0) drain_bar(&q_full[0], 0);
        if (T1.J > 0) drain_bar(&q_full[1], 0);
        for (int i = (kn > KS ? kn - KS : 0); i < kn; ++i) drain_bar(&kfull[i % KS], (i / KS) & 1);
        for (int i = (vn > VS ? vn - VS : 0); i < vn; ++i) drain_bar(&vfull[i % VS], (i / VS) & 1);
      }
    }
   } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------------- MMA issuers
    // Warp 9 issues tile 0's products, warp 10 tile 1's, each in its tile's
    // own order: S_t of block j+1 as soon as S_t of block j has been read
    // (separate P) or O_t += P_t V_j has completed (P under S), O_t += P_t V_j
    // as soon as P_t is written. Every wait is a (bounded) mbarrier try_wait,
    // which suspends the warp in hardware instead of spending issue slots;
    // the leader lane issues from precomputed descriptors.
    const int t = warp - 9;
    const int J = t ? T1.J : T0.J, J_kept = t ? T1.J_kept : T0.J_kept;
    const uint32_t id_qk = idesc_bf16(128, 128, 0);
    const uint32_t id_qk64 = idesc_bf16(128, 64, 0);
    const uint32_t id_pv = idesc_bf16(128, D, 1);
    // Descriptor templates: the start address sits in the low 14 bits (in
    // 16-byte units), so a tile or a K step is a small constant added to the
    // low word; every product's descriptors cost one add each.
    const uint64_t qd = sdesc(su32(sQ), 16, 1024) + (uint64_t)((t * Cfg::kTileBytes) >> 4);
    const uint64_t kd0 = sdesc(su32(sK), 16, 1024);
    const uint64_t vd0 = sdesc(su32(sV), Cfg::kSubBytes, 1024);
    const uint32_t s_tmem = tmem + (uint32_t)(t * 128);
    const uint32_t p_tmem = tmem + Cfg::kPCol + (uint32_t)(t * Cfg::kPStride);
    const uint32_t o_tmem = tmem + Cfg::kOCol + (uint32_t)(t * D);
    const bool leader = elect_one();
    auto wait_all = [&](uint64_t* b, uint32_t parity) -> bool {
      const bool r = __all_sync(0xffffffffu, wait_bar(b, parity, limit, abort_flag));
      if (r) tc_fence_after();
      return r;
    };
    // S_t = Q_t K_j^T (block j in ring entry r), then the commits
    auto issue_qk = [&](int j, int r) {
      if (leader) {
        const uint64_t kd = kd0 + (uint64_t)(((r % KS) * Cfg::kTileBytes) >> 4);
        if (j < J_kept) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * Cfg::kSubBytes + (kk & 3) * 32) >> 4);
            mma_ss(s_tmem, qd + off, kd + off, id_qk, kk > 0 ? 1u : 0u);
          }
        } else {
          // centroid hi parts (rows 0-63), then lo parts (rows 64-127)
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t off = (uint64_t)(((kk >> 2) * Cfg::kSubBytes + (kk & 3) * 32) >> 4);
              mma_ss(s_tmem, qd + off, kd + off + (uint64_t)((half * 64 * 128) >> 4), id_qk64,
                     (half > 0 || kk > 0) ? 1u : 0u);
            }
          }
        }
        tc_commit(&s_full[t]);
        tc_commit(&kempty[r % KS]);
      }
      __syncwarp();
    };
    // O_t += P_t V_j (block j in ring entry r), then the commits
    auto issue_pv = [&](int j, int r) {
      if (leader) {
        const uint64_t vd = vd0 + (uint64_t)(((r % VS) * Cfg::kTileBytes) >> 4);
        if (j < J_kept) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(o_tmem, p_tmem + kk * 8, vd + (uint64_t)((kk * 16 * 128) >> 4), id_pv, (j > 0 || kk > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts(o_tmem, p_tmem + kk * 8, vd + (uint64_t)((half * 64 * 128 + kk * 16 * 128) >> 4), id_pv,
                     (j > 0 || half > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc_commit(&pv_done[t]);
        tc_commit(&vempty[r % VS]);
      }
      __syncwarp();
    };
    auto qk_step = [&](int j) -> bool {
      const int r = ring_of(t, j);
      if (!wait_all(&kfull[r % KS], (r / KS) & 1)) return false;
      issue_qk(j, r);
      return true;
    };
    bool ok = J == 0 || wait_all(&q_full[t], 0);
    if (ok && J > 0) ok = qk_step(0);
    for (int j = 0; ok && j < J; ++j) {
      // separate P: S_t of block j+1 may overwrite S_t of block j once it was read
      if (!Cfg::kAliasP && j + 1 < J) {
        if (!(ok = wait_all(&s_free[t], j & 1))) break;
        if (!(ok = qk_step(j + 1))) break;
      }
      const int r = ring_of(t, j);
      if (!(ok = wait_all(&p_full[t], j & 1))) break;
      if (!(ok = wait_all(&vfull[r % VS], (r / VS) & 1))) break;
      issue_pv(j, r);
      // P under S: S_t of block j+1 waits for O_t += P_t V_j to complete
      if (Cfg::kAliasP && j + 1 < J) {
        if (!(ok = wait_all(&pv_done[t], j & 1))) break;
        if (!(ok = qk_step(j + 1))) break;
      }
    }
    // Drain: every MMA this warp issued has completed once its barrier flips.
    tc_commit_elect(&drain[t]);
    if (lane == 0) drain_bar(&drain[t], 0);
    __syncwarp();
   }
  } else {
    // ------------------------------------------------------------- softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(Cfg::kRegSoftmax));
    constexpr unsigned kPoly = D == 64 ? (unsigned)CA_TC_POLY64 : (unsigned)CA_TC_POLY128;
    const int t = warp >> 2;
    const Tile Tt = make_tile(p, t, p.pair ? kq_union[t] : 0);
    const int q4 = warp & 3;                  // TMEM lane quarter of this warp
    const int grp = p.pair ? (q4 >> 1) : 0;   // pair mode: rows 64-127 belong to the second query cluster
    const int row = q4 * 32 + lane;           // row of the query tile
    const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
    const uint32_t s_addr = lane_addr + (uint32_t)(t * 128);
    const uint32_t p_addr = lane_addr + Cfg::kPCol + (uint32_t)(t * Cfg::kPStride);
    const uint32_t o_addr = lane_addr + Cfg::kOCol + (uint32_t)(t * D);
    const float sc = p.scale_log2;
    float* bias = bias_w + warp * 64;
    // (a tile holding one cluster only: its second half's rows are discarded,
    // and read the first cluster's row)
    const uint32_t* kb_row =
        p.dense ? nullptr : p.kept_bits + ((size_t)Tt.bh * p.C + Tt.a + (Tt.two ? grp : 0)) * ((p.Ck + 31) / 32);
    // the tile's kept clusters' sizes: staged in shared memory, or read through the kept list
    const bool ksm = !p.dense && (p.pair || Tt.kq <= Cfg::kMaxKept);
    const int32_t* kcnt_t = kcnt_s + t * Cfg::kMaxKept;
    const int32_t* kept_t = p.dense ? nullptr : p.kept_idx + ((size_t)Tt.bh * p.C + Tt.a) * p.k;
    const int32_t* cnt_h = p.count_k + (size_t)Tt.bh * p.Ck;
    // members of the kept cluster i for this thread's rows (in pair mode only
    // the clusters its own query cluster keeps; the others are masked)
    auto cnt_of = [&](int i) -> int {
      if (!ksm) return cnt_h[kept_t[i]];
      const int e = kcnt_t[i];
      return (!p.pair || ((e >> (16 + grp)) & 1)) ? (e & 0xFFFF) : 0;
    };
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    // P_t and O_t of the previous block are free once its PV completed
    // (with P under S this is implied by S_t having been computed)
    auto wait_prev_pv = [&](int j) -> bool {
      if (Cfg::kAliasP || j == 0) return true;
      const bool r = __all_sync(0xffffffffu, wait_bar(&pv_done[t], (j - 1) & 1, limit, abort_flag));
      if (r) tc_fence_after();
      return r;
    };
    // O_t holds blocks 0..j-1: scale it when the reference maximum moved
    auto rescale_o = [&](int j, bool need, float factor) {
      if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t ov[32];
          CA_TMEM_LD32(o_addr + (uint32_t)c0, ov);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * factor);
          CA_TMEM_ST32(o_addr + (uint32_t)c0, ov);
        }
      }
    };
    for (int j = 0; j < Tt.J; ++j) {
      const bool cent = j >= Tt.J_kept;
      int v0 = 64, v1 = 64;   // real keys in the two 64-column halves of a kept block
      if (cent) {
        // compensation bias of this block's 64 centroids (log2 units; -inf
        // where the key cluster is kept or is padding), staged per warp
        const float log2e = 1.4426950408889634f;
        __syncwarp();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int e = h * 32 + lane;
          const int b = (j - Tt.J_kept) * 64 + e;
          float bv = -INFINITY;
          if (b < p.Ck && !((kb_row[b >> 5] >> (b & 31)) & 1u)) bv = p.logcnt[(size_t)Tt.bh * p.Cpad + b] * log2e;
          bias[e] = bv;
        }
        __syncwarp();
      } else if (p.dense) {
        const int rem = p.n_valid - j * 128;
        v0 = min(max(rem, 0), 64);
        v1 = min(max(rem - 64, 0), 64);
      } else if (p.ck >= 128) {
        // c_k is 128 or 256: one or two key blocks per kept cluster (shifts,
        // not a division, on the softmax warps' path)
        const int sh = p.ck >> 8;
        const int rem = cnt_of(j >> sh) - (j & sh) * 128;
        v0 = min(max(rem, 0), 64);
        v1 = min(max(rem - 64, 0), 64);
      } else {
        v0 = cnt_of(2 * j);
        v1 = (2 * j + 1 < Tt.kq) ? cnt_of(2 * j + 1) : 0;
      }
      ok = __all_sync(0xffffffffu, wait_bar(&s_full[t], j & 1, limit, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float factor;
      bool need;
      if (cent) {
        float v[64];
        uint32_t pk[32];
        CA_TMEM_LD32(s_addr, reinterpret_cast<uint32_t*>(v));
        CA_TMEM_LD32(s_addr + 32u, reinterpret_cast<uint32_t*>(v + 32));
        tmem_wait_ld();
        if (!Cfg::kAliasP) { tc_fence_before(); mbar_arrive(&s_free[t]); }
        need = softmax_block<64, kPoly>(v, pk, sc, bias, 64, 0, m_ref, l, factor);
        if (!(ok = wait_prev_pv(j))) break;
        CA_TMEM_ST32(p_addr, pk);
      } else {
        float v[128];
        uint32_t pk[64];
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) CA_TMEM_LD32(s_addr + (uint32_t)c0, reinterpret_cast<uint32_t*>(v + c0));
        tmem_wait_ld();
        if (!Cfg::kAliasP) { tc_fence_before(); mbar_arrive(&s_free[t]); }
        need = softmax_block<128, kPoly>(v, pk, sc, nullptr, v0, v1, m_ref, l, factor);
        if (!(ok = wait_prev_pv(j))) break;
        CA_TMEM_ST32(p_addr, pk);
        CA_TMEM_ST32(p_addr + 32u, (pk + 32));
      }
      rescale_o(j, need, factor);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    // epilogue: O / l to the query's original row (zero when the tile had no
    // block at all: nothing kept and no compensation)
    if (ok && Tt.exists) {
      if (Tt.J > 0) ok = __all_sync(0xffffffffu, wait_bar(&pv_done[t], (Tt.J - 1) & 1, limit, abort_flag));
      if (ok) {
        if (Tt.J > 0) tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        int orow;
        if (p.dense) orow = Tt.qrow + row < p.n_valid ? Tt.qrow + row : -1;
        else if (p.pair) orow = row < (Tt.two ? 128 : 64) ? p.perm_q[(size_t)Tt.qrow + row] : -1;
        else orow = (Tt.sub * 128 + row < p.c && row < p.rows_per_tile) ? p.perm_q[(size_t)Tt.qrow + row] : -1;
        __nv_bfloat16* dst = p.O + p.TL.head(Tt.bh) + (size_t)(orow < 0 ? 0 : orow) * p.TL.sn;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          if (Tt.J > 0) {
            CA_TMEM_LD32(o_addr + (uint32_t)c0, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) o[q] = 0u;
          }
          if (orow >= 0) {
            uint4 w[4];
            uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
            for (int q = 0; q < 16; ++q) wp[q] = pack_bf16(__uint_as_float(o[2 * q]) * inv, __uint_as_float(o[2 * q + 1]) * inv);
            uint4* gp = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) gp[q] = w[q];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(Cfg::kTmemCols));
  }
}

// Evaluates exp2_poly2 on n inputs (pairs), for checking it against exp2f.
__global__ void exp2_poly_check_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float t0 = x[i], t1 = i + 1 < n ? x[i + 1] : 0.f;
  float r0, r1;
  exp2_poly2(t0, t1, r0, r1);
  y[i] = r0;
  if (i + 1 < n) y[i + 1] = r1;
}

// ---------------------------------------------------------------------------
// Host: tensor maps and launch
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2-D bf16 map over [rows][D], box {64, box_rows}, 128-byte swizzle.
bool make_map_2d(CUtensorMap* m, const void* base, uint64_t rows, int D, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)D, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// 4-D bf16 map over the caller's tensor exposing only tokens < n_valid of
// each head: dimensions (d, tokens, heads, batch) when consecutive tokens of
// a head are closer than consecutive heads (CA_LAYOUT_BHND), else (d, heads,
// tokens, batch) (CA_LAYOUT_BNHD), so the strides increase; a box is 64
// columns of 128 tokens of one head either way.
bool make_map_dense(CUtensorMap* m, const void* base, const ca_shape* s, bool* tok_inner) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const TensorLayout L = tensor_layout(s);
  const bool ti = L.sn <= L.sh;
  *tok_inner = ti;
  const cuuint64_t D = (cuuint64_t)s->d, n = (cuuint64_t)s->n_valid, H = (cuuint64_t)s->H, B = (cuuint64_t)s->B;
  const cuuint64_t dims[4] = {D, ti ? n : H, ti ? H : n, B};
  const cuuint64_t strides[3] = {(cuuint64_t)(ti ? L.sn : L.sh) * 2, (cuuint64_t)(ti ? L.sh : L.sn) * 2,
                                 (cuuint64_t)L.sb * 2};
  const cuuint32_t box[4] = {64, ti ? 128u : 1u, ti ? 1u : 128u, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_tc(const CUtensorMap maps[5], const TcParams& p, dim3 grid, cudaStream_t st) {
  using Cfg = TcCfg<D>;
  // The register split inside the kernel assumes exactly kRegLaunch registers
  // per thread at launch; any other count could leave setmaxnreg.inc waiting.
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, tc_attend_kernel<D>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != Cfg::kRegLaunch) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(tc_attend_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
  if (e != cudaSuccess) return e;
  tc_attend_kernel<D><<<grid, Cfg::kThreads, Cfg::kSmem, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], p);
  return cudaGetLastError();
}

cudaError_t dispatch(int D, const CUtensorMap maps[5], const TcParams& p, dim3 grid, cudaStream_t st) {
  return D == 64 ? launch_tc<64>(maps, p, grid, st) : launch_tc<128>(maps, p, grid, st);
}

}  // namespace

cudaError_t launch_attend_tc(const ca_shape* s, const ca_clusters* cl, const ca_routes* rt, int compensate,
                             void* O, const AttendWs& L, char* ws, cudaStream_t st) {
  const int BH = s->B * s->H, D = s->d, c = s->c, C = L.C, ck = key_c(s), Ck = L.Ck;
  const uint64_t slots_q = (uint64_t)BH * C * c, slots_k = (uint64_t)BH * Ck * ck;
  const uint64_t cent_rows = (uint64_t)BH * L.Cpad * 2;   // hi and lo rows of every 64-centroid block
  CUtensorMap maps[5];
  bool ok = make_map_2d(&maps[0], ws + L.qp, slots_q, D, 128) &&
            make_map_2d(&maps[1], ws + L.kp, slots_k, D, ck >= 128 ? 128 : 64) &&
            make_map_2d(&maps[2], ws + L.vp, slots_k, D, ck >= 128 ? 128 : 64) &&
            make_map_2d(&maps[3], ws + L.kbar_hl, cent_rows, D, 128) &&
            make_map_2d(&maps[4], ws + L.vbar_hl, cent_rows, D, 128);
  if (!ok) return cudaErrorInvalidValue;
  TcParams p{};
  p.C = C; p.c = c; p.Ck = Ck; p.ck = ck;
  p.k = rt->k; p.Cpad = L.Cpad; p.n_valid = s->n_valid; p.N_alloc = s->N_alloc;
  p.TL = tensor_layout(s);
  p.tiles_per_cluster = c >= 128 ? c / 128 : 1;
  p.rows_per_tile = c >= 128 ? 128 : c;
  // 64-query clusters go two to a 128-row tile while their union of kept key
  // clusters (at most 2 k) fits the kernel's staged list
  p.pair = (c == 64 && 2 * rt->k <= 512) ? 1 : 0;
  p.n_tiles = p.pair ? BH * ((C + 1) / 2) : BH * C * p.tiles_per_cluster;
  p.compensate = compensate;
  p.J_cent = compensate ? (Ck + 63) / 64 : 0;
  p.dense = 0;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  p.perm_q = cl->perm_q; p.count_k = cl->count_k; p.kept_idx = rt->kept_idx; p.kept_bits = rt->kept_bits;
  p.kept_count = rt->kept_count;
  p.logcnt = reinterpret_cast<const float*>(ws + L.logcnt);
  p.O = static_cast<__nv_bfloat16*>(O);
  p.wait_limit = wait_limit();
  const dim3 grid((unsigned)((p.n_tiles + 1) / 2));
  return dispatch(D, maps, p, grid, st);
}

// One CTA waits, through the same bounded wait as the attention kernel, on an
// mbarrier that completes only if `arrive` is set: with arrive = 0 nothing
// ever flips it, the wait runs out after limit_ns and raises CA_ERR_TIMEOUT in
// the device error word. Touches no global data besides that word.
__global__ void bounded_wait_check_kernel(uint64_t limit_ns, int arrive) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (arrive) mbar_arrive(&bar);
    wait_bar(&bar, 0, limit_ns, &abort_flag);
  }
}

cudaError_t launch_bounded_wait_check(uint64_t limit_ns, int arrive, cudaStream_t st) {
  bounded_wait_check_kernel<<<1, 32, 0, st>>>(limit_ns, arrive);
  return cudaGetLastError();
}

cudaError_t launch_exp2_poly_check(const float* x, float* y, int n, cudaStream_t st) {
  const int pairs = (n + 1) / 2;
  exp2_poly_check_kernel<<<(pairs + 255) / 256, 256, 0, st>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_dense_tc(const void* Q, const void* K, const void* V, const ca_shape* s, void* O,
                            cudaStream_t st) {
  const int BH = s->B * s->H, D = s->d;
  CUtensorMap maps[5];
  bool ti = true;
  bool ok = make_map_dense(&maps[0], Q, s, &ti) && make_map_dense(&maps[1], K, s, &ti) &&
            make_map_dense(&maps[2], V, s, &ti);
  if (!ok) return cudaErrorInvalidValue;
  maps[3] = maps[1]; maps[4] = maps[2];
  TcParams p{};
  p.TL = tensor_layout(s);
  p.dense_tok_inner = ti ? 1 : 0;
  p.n_valid = s->n_valid; p.N_alloc = s->N_alloc;
  p.tiles_per_cluster = 1; p.rows_per_tile = 128;
  p.compensate = 0; p.J_cent = 0; p.dense = 1;
  p.dense_tiles = (s->n_valid + 127) / 128;
  p.dense_key_blocks = (s->n_valid + 127) / 128;
  p.c = 128; p.ck = 128;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  p.O = static_cast<__nv_bfloat16*>(O);
  p.wait_limit = wait_limit();
  const dim3 grid((unsigned)((p.dense_tiles + 1) / 2), BH);
  return dispatch(D, maps, p, grid, st);
}

}  // namespace ca
