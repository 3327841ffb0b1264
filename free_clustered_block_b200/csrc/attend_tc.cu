// Block-sparse attention with striped mean-compensation on the sm_100a
// tensor cores (tcgen05, TMEM accumulators, TMA tiles).
//
// ClusterAttention paper, Section 3.1 (attention over the kept key clusters
// of each query cluster, blocks of the permuted tokens) and Appendix A,
// eq. 21-22 (every excluded key cluster b enters the softmax with logit
// q . kbar_b / sqrt(d) + ln|b| and value vbar_b). The dense form (eq. 1) is
// the same kernel with every key block kept and no compensation.
//
// One CTA handles one 128-row query tile of one head and holds an SM (512
// TMEM columns: three S buffers and O):
//   warp 0      TMA producer (one thread): Q tile once, then a ring of
//               stages holding (K, V) of a kept key block, (kbar_hi,
//               kbar_lo) or (vbar_hi, vbar_lo) of a centroid block;
//   warp 1      MMA issuer (the converged warp, one elected lane issuing):
//               S_j = Q K_j^T into TMEM buffer j % 3 and O += P_j V_j with
//               P_j read from TMEM. S_{j+2} is issued right behind PV_j: its
//               buffer was last read by PV_{j-1}, so the tensor pipe gets both
//               without waiting for PV_j, and the softmax of S_{j+1} overlaps;
//   warps 2..9  softmax, two threads per query row (one per half of the key
//               block): read S_j from TMEM, apply the key mask /
//               compensation bias, exchange the row max through shared
//               memory, keep a running max (rescaling O only when the max
//               grows by more than 2^8), write P_j as bf16 over the front of
//               S_j, accumulate the row sums in registers, and finally write
//               O / l to the query's original row.
// Centroids are split into bf16 hi + lo parts and enter as two MMAs each.
// Every wait is bounded: on a timeout the CTA sets the library's device error
// word (CA_ERR_TIMEOUT), drains what it issued, frees TMEM and returns.
#include <cuda.h>

#include "ca_internal.cuh"

namespace ca {

__device__ unsigned int g_device_error = 0;
static uint64_t g_wait_limit = 0;
// Bounded waits are timed with the global nanosecond timer.
constexpr uint64_t kDefaultWaitLimit = 1000000000ull;   // 1 s
// Drains (letting copies and MMAs already issued finish before the CTA
// leaves) use their own bound, independent of the adjustable wait limit.
constexpr uint64_t kDrainLimitNs = 1000000000ull;

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
__device__ __forceinline__ void tma_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(su32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(su32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// tcgen05.mma (A and B from shared memory, or A from TMEM) and commit, issued
// by one elected lane of a converged warp: the whole warp computes the
// (warp-uniform) operands, so issue needs no divergent single-lane code.
__device__ __forceinline__ void mma_ss_elect(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p, e;\n setp.ne.b32 p, %4, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(0u)
      : "memory");
}
__device__ __forceinline__ void mma_ts_elect(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p, e;\n setp.ne.b32 p, %4, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n}\n" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc), "r"(0u)
      : "memory");
}
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
// 2^t0, 2^t1 (t <= 8) on the FMA pipe, to take part of the load off the
// MUFU ex2 unit: t = n + f with n = round(t) (adding and subtracting 1.5 * 2^23
// leaves the rounded integer in the low mantissa bits), 2^f on [-1/2, 1/2] by
// a cubic fitted to the least maximum relative error on that interval
// (< 8e-5, far below the bf16 rounding of P), and n added into the exponent
// field with one integer multiply-add. t is clamped at -126 (2^-126 is as good
// as 0 in a bf16 P).
__device__ __forceinline__ void exp2_poly2(float t0, float t1, float& r0, float& r1) {
  constexpr float kRound = 12582912.f;   // 1.5 * 2^23
  constexpr float c0 = 0.9999281168f, c1 = 0.6932609677f, c2 = 0.2426105440f, c3 = 0.0551713221f;
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
  // low mantissa bits of y hold n (two's complement); times 2^23 moves them to the exponent
  r0 = __int_as_float(__float_as_int(y0) * 8388608 + __float_as_int(q0));
  r1 = __int_as_float(__float_as_int(y1) * 8388608 + __float_as_int(q1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
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
__device__ __noinline__ bool wait_bar_slow(uint64_t* b, uint32_t parity, uint64_t limit_ns,
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
// The first probe is inline: a barrier that has already flipped costs no call.
__device__ __forceinline__ bool wait_bar(uint64_t* b, uint32_t parity, uint64_t limit_ns, volatile int* abort_flag) {
  if (mbar_try(b, parity)) return true;
  return wait_bar_slow(b, parity, limit_ns, abort_flag);
}
// Bounded wait used while draining: ignores the abort flag, fixed limit.
__device__ __noinline__ void drain_bar(uint64_t* b, uint32_t parity) {
  const uint64_t t0 = now_ns();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try(b, parity)) return;
    if ((i & 31) == 31 && now_ns() - t0 > kDrainLimitNs) return;
  }
}

// ---------------------------------------------------------------------------
// Kernel parameters
// ---------------------------------------------------------------------------
struct TcParams {
  int C, c, k, Cpad, n_valid, N_alloc;
  int tiles_per_cluster;      // c / 128 (>= 1)
  int rows_per_tile;          // min(c, 128)
  int compensate;
  int dense;                  // 1: identity order, every key block kept
  int dense_key_blocks;       // ceil(n_valid / KB) in dense mode
  float scale_log2;           // log2(e) / sqrt(d)
  const int32_t* perm_q;      // [BH][C*c]
  const int32_t* count_k;     // [BH][C]
  const int32_t* kept_idx;    // [BH][C][k]
  const int32_t* kept_count;  // [BH][C] kept per query cluster, or null (k each)
  const uint32_t* kept_bits;  // [BH][C][W]
  const float* logcnt;        // [BH][Cpad] natural log of counts
  __nv_bfloat16* O;           // [BH][N_alloc][D]
  uint64_t wait_limit;
};

template <int D, int KB>
struct TcCfg {
  static constexpr int kSub = D / 64;                                  // 64-column sub-tiles per row
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kTileBytes = KB * D * 2;                        // one K (or V) block
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kMaxKeptSmem = 1024;                            // kept list staged in shared memory
  static constexpr int kMaxBias = 8192;                                // centroid columns (C <= 8192)
  static constexpr int kFixedBytes = 256 + kMaxBias * 4 + 2 * 2 * 128 * 4 + 2 * kMaxKeptSmem * 4 + 1024;
  static constexpr int kStagesFit = (200 * 1024 - kQBytes - kFixedBytes) / kStageBytes;
  static constexpr int kStages = kStagesFit > 4 ? 4 : (kStagesFit < 2 ? 2 : kStagesFit);
  static constexpr int kBarOff = kQBytes + kStages * kStageBytes;
  static constexpr int kBiasOff = kBarOff + 256;                       // compensation bias per centroid column
  static constexpr int kXchOff = kBiasOff + kMaxBias * 4;              // (m, l) exchange [2 groups][2][128]
  static constexpr int kKeptOff = kXchOff + 2 * 2 * 128 * 4;
  // + alignment slack; at least 116 KB so that one CTA (and its 512 TMEM
  // columns) holds an SM
  static constexpr int kSmemCalc = kKeptOff + 2 * kMaxKeptSmem * 4 + 1024;
  static constexpr int kSmem = kSmemCalc > 116 * 1024 ? kSmemCalc : 116 * 1024;
  static constexpr int kGroupThreads = 128;                            // one softmax group: a thread per row
  static constexpr int kSoftmaxThreads = 2 * kGroupThreads;
  static constexpr int kThreads = 128 + kSoftmaxThreads;               // warps 0-3: producer, MMA, 2 idle
  static constexpr uint32_t kTmemCols = 512;
  // TMEM: NB S buffers of KB columns (P_j as bf16 pairs over the front half
  // of its buffer), then O_0 and O_1 (fp32, D columns each)
  static constexpr int kNBufFit = (512 - 2 * D) / KB;
  // S_{j+NB} is issued after PV_j; a centroid block takes two stages (kbar,
  // then vbar), so the stage S_{j+NB} needs is free by then only while
  // NB <= floor(stages / 2) + 1 (otherwise it waits on a PV not yet issued)
  static constexpr int kNBufPipe = kStages / 2 + 1;
  static constexpr int kNBuf = kNBufFit < kNBufPipe ? kNBufFit : kNBufPipe;
  static constexpr int kSPhase = (kNBuf % 2 == 0) ? kNBuf : 2 * kNBuf;   // blocks between uses of one s_full
  static constexpr uint32_t kSCol = 0;
  static constexpr uint32_t kOCol = kNBuf * KB;
  static_assert(kNBuf >= 2, "two S buffers at least");
  static_assert(kNBuf <= kStages / 2 + 1 && kNBuf <= kStages, "S look-ahead must not outrun the stage ring");
  static_assert(kOCol + 2 * D <= kTmemCols, "S buffers and both O accumulators must fit in TMEM");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

// Pairs of P columns (bit q % 8) whose exponentials run on the FMA pipe
// instead of the MUFU unit.
#ifndef CA_TC_POLY_PAIRS
#define CA_TC_POLY_PAIRS 0x00
#endif
constexpr unsigned kPolyPairs = CA_TC_POLY_PAIRS;

// Items in load order: kept key sub-blocks (K,V), then per centroid block
// (kbar hi, lo) and (vbar hi, vbar lo).
struct Item { int kind; int row; };   // kind 0 KV, 1 KBAR, 2 VBAR

template <int D, int KB>
__global__ void __launch_bounds__(TcCfg<D, KB>::kThreads, 1)
tc_attend_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_khi,
                 const __grid_constant__ CUtensorMap tm_klo, const __grid_constant__ CUtensorMap tm_vhi,
                 const __grid_constant__ CUtensorMap tm_vlo, const TcParams p) {
  using Cfg = TcCfg<D, KB>;
  constexpr int NS = Cfg::kStages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  unsigned char* sQ = smem;
  unsigned char* sStage = smem + Cfg::kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* full = bars;              // [NS] stage loaded
  uint64_t* empty = bars + NS;        // [NS] stage released
  uint64_t* q_full = bars + 2 * NS;   // Q tile loaded
  constexpr int NB = Cfg::kNBuf;
  uint64_t* s_full = q_full + 1;      // [NB][2] S_j computed in buffer j % NB, for group j % 2
  uint64_t* p_full = s_full + 2 * NB; // [NB] P_j written in buffer j % NB
  uint64_t* pv_done = p_full + NB;    // [NB] O_{j%2} += P_j V_j completed (j % NB)
  uint64_t* drain = pv_done + NB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* bias_all = reinterpret_cast<float*>(smem + Cfg::kBiasOff);
  float* xch = reinterpret_cast<float*>(smem + Cfg::kXchOff);
  int32_t* kept_s = reinterpret_cast<int32_t*>(smem + Cfg::kKeptOff);        // kept key clusters
  int32_t* kcnt_s = kept_s + Cfg::kMaxKeptSmem;                               // their member counts

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int tile = blockIdx.x;
  const int a = p.dense ? 0 : tile / p.tiles_per_cluster;          // query cluster
  const int sub_tile = p.dense ? 0 : tile % p.tiles_per_cluster;
  const int nsb = p.dense ? 1 : (p.c + KB - 1) / KB;               // key sub-blocks per cluster
  // kept key clusters of this query cluster (k, or its own count after adaptive selection)
  const int kq = p.dense ? 0 : (p.kept_count ? min(max(p.kept_count[(size_t)bh * p.C + a], 0), p.k) : p.k);
  const int J_kept = p.dense ? p.dense_key_blocks : kq * nsb;
  const int J_cent = (p.compensate && !p.dense) ? p.Cpad / KB : 0;
  const int J = J_kept + J_cent;
  const int n_items = J_kept + 2 * J_cent;
  const int32_t* kept_g = p.dense ? nullptr : p.kept_idx + ((size_t)bh * p.C + a) * p.k;
  const bool kept_in_smem = !p.dense && kq <= Cfg::kMaxKeptSmem;
  if (kept_in_smem) {
    for (int i = threadIdx.x; i < kq; i += Cfg::kThreads) {
      const int b = kept_g[i];
      kept_s[i] = b;
      kcnt_s[i] = p.count_k[(size_t)bh * p.C + b];
    }
  }
  const int32_t* kept = kept_in_smem ? kept_s : kept_g;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(q_full, 1);
    for (int b = 0; b < NB; ++b) {
      mbar_init(&s_full[2 * b], 1);
      mbar_init(&s_full[2 * b + 1], 1);
      mbar_init(&p_full[b], Cfg::kGroupThreads);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(drain, 1);
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

  auto item_of = [&](int i) -> Item {
    Item it;
    if (i < J_kept) {
      it.kind = 0;
      if (p.dense) it.row = i * KB;
      else {
        const int b = kept[i / nsb];
        it.row = (bh * p.C + b) * p.c + (i % nsb) * KB;
      }
    } else {
      const int t = i - J_kept;
      it.kind = 1 + (t & 1);
      it.row = bh * p.Cpad + (t >> 1) * KB;
    }
    return it;
  };

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      mbar_expect_tx(q_full, Cfg::kQBytes);
      for (int s = 0; s < Cfg::kSub; ++s) {
        if (p.dense) tma_3d(sQ + s * 128 * 128, &tm_q, q_full, s * 64, tile * 128, bh);
        else tma_2d(sQ + s * 128 * 128, &tm_q, q_full, s * 64, (bh * p.C + a) * p.c + sub_tile * 128);
      }
      for (int i = 0; i < n_items && ok; ++i) {
        const int s = i % NS, r = i / NS;
        const Item it = item_of(i);
        if (!wait_bar(&empty[s], (r & 1) ^ 1, limit, abort_flag)) { ok = false; break; }
        unsigned char* dst = sStage + s * Cfg::kStageBytes;
        mbar_expect_tx(&full[s], Cfg::kStageBytes);
        const CUtensorMap* m0 = it.kind == 0 ? &tm_k : (it.kind == 1 ? &tm_khi : &tm_vhi);
        const CUtensorMap* m1 = it.kind == 0 ? &tm_v : (it.kind == 1 ? &tm_klo : &tm_vlo);
        for (int sb = 0; sb < Cfg::kSub; ++sb) {
          if (p.dense) {
            tma_3d(dst + sb * KB * 128, m0, &full[s], sb * 64, it.row, bh);
            tma_3d(dst + Cfg::kTileBytes + sb * KB * 128, m1, &full[s], sb * 64, it.row, bh);
          } else {
            tma_2d(dst + sb * KB * 128, m0, &full[s], sb * 64, it.row);
            tma_2d(dst + Cfg::kTileBytes + sb * KB * 128, m1, &full[s], sb * 64, it.row);
          }
        }
        issued = i + 1;
      }
      if (!ok) {
        // Let every copy already issued land before the CTA leaves.
        drain_bar(q_full, 0);
        for (int i = (issued > NS ? issued - NS : 0); i < issued; ++i) drain_bar(&full[i % NS], (i / NS) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    // The whole warp runs this loop (so descriptors are warp-uniform); one
    // elected lane issues each tcgen05 instruction and every commit.
    constexpr uint32_t id_qk = idesc_bf16(128, KB, 0);
    constexpr uint32_t id_pv = idesc_bf16(128, D, 1);
    const uint32_t q_base = su32(sQ);
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, wait_bar(bar, parity, limit, abort_flag));
    };
    bool ok = wwait(q_full, 0);
    // item index of block j's QK and PV operands
    auto qk_item = [&](int j) { return j < J_kept ? j : J_kept + 2 * (j - J_kept); };
    auto pv_item = [&](int j) { return j < J_kept ? j : J_kept + 2 * (j - J_kept) + 1; };
    auto issue_qk = [&](int j) -> bool {
      const int i = qk_item(j);
      const int s = i % NS, r = i / NS;
      if (!wwait(&full[s], r & 1)) return false;
      tc_fence_after();
      const uint32_t kb = su32(sStage + s * Cfg::kStageBytes);
      const uint32_t d_tmem = tmem + Cfg::kSCol + (uint32_t)((j % NB) * KB);
      const int nmat = (j < J_kept) ? 1 : 2;   // centroids: hi then lo
      for (int mtx = 0; mtx < nmat; ++mtx) {
        const uint32_t bbase = kb + mtx * Cfg::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)((kk & 3) * 32);   // 16 bf16 along K inside the 128B row
          const uint64_t ad = sdesc(q_base + (kk >> 2) * 128 * 128 + off, 16, 1024);
          const uint64_t bd = sdesc(bbase + (kk >> 2) * KB * 128 + off, 16, 1024);
          mma_ss_elect(d_tmem, ad, bd, id_qk, (mtx > 0 || kk > 0) ? 1u : 0u);
        }
      }
      tc_commit_elect(&s_full[(j % NB) * 2 + (j & 1)]);
      if (j >= J_kept) tc_commit_elect(&empty[s]);   // kbar stage is free once S is computed
      return true;
    };
    // S_0 .. S_{NB-1} ahead; S_{j+NB} reuses buffer j % NB once PV_j (its
    // last reader) has completed. Blocks alternate between the two softmax
    // groups, so the other group works on S_{j+1} meanwhile.
    for (int j = 0; j < NB && j < J && ok; ++j) ok = issue_qk(j);
    for (int j = 0; j < J && ok; ++j) {
      if (!wwait(&p_full[j % NB], (j / NB) & 1)) { ok = false; break; }
      tc_fence_after();
      const int i = pv_item(j);
      const int s = i % NS, r = i / NS;
      if (j >= J_kept) {
        if (!wwait(&full[s], r & 1)) { ok = false; break; }
        tc_fence_after();
      }
      const uint32_t vb = su32(sStage + s * Cfg::kStageBytes) + (j < J_kept ? Cfg::kTileBytes : 0);
      const uint32_t p_tmem = tmem + Cfg::kSCol + (uint32_t)((j % NB) * KB);
      const uint32_t o_tmem = tmem + Cfg::kOCol + (uint32_t)((j & 1) * D);   // O of the block's group
      const int nmat = (j < J_kept) ? 1 : 2;
      for (int mtx = 0; mtx < nmat; ++mtx) {
        const uint32_t bbase = vb + mtx * Cfg::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < KB / 16; ++kk) {
          const uint64_t bd = sdesc(bbase + kk * 16 * 128, KB * 128, 1024);
          mma_ts_elect(o_tmem, p_tmem + kk * 8, bd, id_pv, (j >= 2 || mtx > 0 || kk > 0) ? 1u : 0u);
        }
      }
      tc_commit_elect(&pv_done[j % NB]);
      tc_commit_elect(&empty[s]);
      if (j + NB < J) {
        if (!wwait(&pv_done[j % NB], (j / NB) & 1)) { ok = false; break; }
        tc_fence_after();
        if (!issue_qk(j + NB)) { ok = false; break; }
      }
    }
    // Drain: every MMA issued so far has completed once `drain` flips.
    tc_commit_elect(drain);
    if (lane == 0) drain_bar(drain, 0);
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------- softmax
    // Group g (warps 4-7 or 8-11) takes the blocks j with j % 2 == g, one
    // thread per query row, and accumulates them in its own O_g.
    const int g = (warp - 4) >> 2;
    const int q4 = warp & 3;                  // TMEM lane quarter of this warp
    const int row = q4 * 32 + lane;           // row of the query tile
    const int sth = threadIdx.x - 128;        // 0..255 over both groups
    const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
    const float sc = p.scale_log2;
    // compensation bias of every centroid column (log2 units; -inf where the
    // key cluster is kept or is padding), once per CTA
    if (J_cent > 0) {
      const uint32_t* kb_row = p.kept_bits + ((size_t)bh * p.C + a) * ((p.C + 31) / 32);
      const float log2e = 1.4426950408889634f;
      for (int e = sth; e < J_cent * KB; e += Cfg::kSoftmaxThreads) {
        float bv = -INFINITY;
        if (e < p.C && !((kb_row[e >> 5] >> (e & 31)) & 1u)) bv = p.logcnt[(size_t)bh * p.Cpad + e] * log2e;
        bias_all[e] = bv;
      }
    }
    named_sync(1, Cfg::kSoftmaxThreads);
    float m_used = -INFINITY, lreg = 0.f;
    bool ok = true;
    for (int j = g; j < J; j += 2) {
      const bool cent = j >= J_kept;
      int valid = KB;   // real keys in a kept block
      if (!cent) {
        if (p.dense) valid = min(KB, p.n_valid - j * KB);
        else {
          const int cnt = kept_in_smem ? kcnt_s[j / nsb] : p.count_k[(size_t)bh * p.C + kept[j / nsb]];
          valid = min(KB, cnt - (j % nsb) * KB);
        }
      }
      const float* bias = bias_all + (cent ? (j - J_kept) * KB : 0);
      const uint32_t sbuf = lane_addr + Cfg::kSCol + (uint32_t)((j % NB) * KB);
      ok = __all_sync(0xffffffffu, wait_bar(&s_full[(j % NB) * 2 + g], (j / Cfg::kSPhase) & 1, limit, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // pass 1: the row maximum, 64 columns per TMEM round trip. Partial and
      // centroid blocks (rare) get their mask / bias here and are written
      // back, so that pass 2 has a single path.
      const bool special = cent || valid < KB;
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
#pragma unroll 1
      for (int c0 = 0; c0 < KB; c0 += 64) {
        float v[64];
        CA_TMEM_LD32(sbuf + (uint32_t)c0, reinterpret_cast<uint32_t*>(v));
        CA_TMEM_LD32(sbuf + (uint32_t)(c0 + 32), reinterpret_cast<uint32_t*>(v + 32));
        tmem_wait_ld();
        if (special) {
          if (cent) {
#pragma unroll
            for (int q = 0; q < 64; ++q) v[q] = fmaf(v[q], sc, bias[c0 + q]);
          } else {
#pragma unroll
            for (int q = 0; q < 64; ++q) v[q] = (c0 + q < valid) ? v[q] : -INFINITY;
          }
          CA_TMEM_ST32(sbuf + (uint32_t)c0, reinterpret_cast<uint32_t*>(v));
          CA_TMEM_ST32(sbuf + (uint32_t)(c0 + 32), reinterpret_cast<uint32_t*>(v + 32));
        }
#pragma unroll
        for (int q = 0; q < 64; q += 2) m8[(q >> 1) & 7] = max3(m8[(q >> 1) & 7], v[q], v[q + 1]);
      }
      if (special) tmem_wait_st();
      float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      if (!cent) mx *= sc;                   // log2 units (centroid values already are)
      // lazy rescale: move the reference max only when it grows by > 8 (x 256)
      float factor = 1.f;
      const bool need = mx > m_used + 8.f;
      if (need) {
        factor = (m_used == -INFINITY) ? 0.f : ex2(m_used - mx);
        m_used = mx;
        lreg *= factor;
      }
      // O_g already holds blocks j-2, j-4, ...: rescale it (whole warp, as
      // TMEM loads and stores are warp-wide) once PV_{j-2} has completed.
      if (j >= 2 && __any_sync(0xffffffffu, need)) {
        ok = __all_sync(0xffffffffu, wait_bar(&pv_done[(j - 2) % NB], ((j - 2) / NB) & 1, limit, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const uint32_t oaddr = lane_addr + Cfg::kOCol + (uint32_t)(g * D);
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t ov[32];
          CA_TMEM_LD32(oaddr + (uint32_t)c0, ov);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * factor);
          CA_TMEM_ST32(oaddr + (uint32_t)c0, ov);
        }
      }
      const float nb = (m_used == -INFINITY) ? 0.f : -m_used;
      // pass 2: P = 2^(x - m) as bf16 pairs over the front half of the buffer
      // (the pairs of columns c0.. land on columns c0/2.., already read)
      const float xs = cent ? 1.f : sc;
      const uint64_t xs2 = f2_pack(xs, xs), nb2 = f2_pack(nb, nb);
      uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};   // packed partial row sums
      // 32 columns per step, two steps per loop turn; the next step's TMEM
      // load is in flight while a step computes
      auto p_step = [&](const float* v, int c0) {
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float t0, t1, p0, p1;
          f2_unpack(fma2(f2_pack(v[2 * q], v[2 * q + 1]), xs2, nb2), t0, t1);
          if ((kPolyPairs >> (q & 7)) & 1) exp2_poly2(t0, t1, p0, p1);
          else { p0 = ex2(t0); p1 = ex2(t1); }
          ls2[q & 3] = add2(ls2[q & 3], f2_pack(p0, p1));
          pk[q] = pack_bf16(p0, p1);
        }
        CA_TMEM_ST16(sbuf + (uint32_t)(c0 / 2), pk);
      };
      float va[32], vb[32];
      CA_TMEM_LD32(sbuf, reinterpret_cast<uint32_t*>(va));
#pragma unroll 1
      for (int c0 = 0; c0 < KB; c0 += 64) {
        tmem_wait_ld();
        CA_TMEM_LD32(sbuf + (uint32_t)(c0 + 32), reinterpret_cast<uint32_t*>(vb));
        p_step(va, c0);
        tmem_wait_ld();
        if (c0 + 64 < KB) CA_TMEM_LD32(sbuf + (uint32_t)(c0 + 64), reinterpret_cast<uint32_t*>(va));
        p_step(vb, c0 + 32);
      }
      {
        float a0, a1;
        f2_unpack(add2(add2(ls2[0], ls2[1]), add2(ls2[2], ls2[3])), a0, a1);
        lreg += a0 + a1;
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[j % NB]);
    }
    // epilogue: merge the two groups' (m, l, O) and write O / l to the
    // query's original row; group g writes columns [g D/2, (g+1) D/2)
    const int jl0 = (J >= 1) ? ((J - 1) & ~1) : -1;          // last block of group 0
    const int jl1 = (J >= 2) ? (((J - 2) & ~1) + 1) : -1;    // last block of group 1
    const int jl = g ? jl1 : jl0;
    if (ok && jl >= 0)
      ok = __all_sync(0xffffffffu, wait_bar(&pv_done[jl % NB], (jl / NB) & 1, limit, abort_flag));
    xch[(g * 2 + 0) * 128 + row] = jl >= 0 ? m_used : -INFINITY;
    xch[(g * 2 + 1) * 128 + row] = jl >= 0 ? lreg : 0.f;
    named_sync(1, Cfg::kSoftmaxThreads);
    if (ok) {
      tc_fence_after();
      const float m0 = xch[0 * 128 + row], l0 = xch[1 * 128 + row];
      const float m1 = xch[2 * 128 + row], l1 = xch[3 * 128 + row];
      const float M = fmaxf(m0, m1);
      const float f0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M);
      const float f1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M);
      const float l = l0 * f0 + l1 * f1;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float w0 = f0 * inv, w1 = f1 * inv;
      int orow;
      if (p.dense) orow = tile * 128 + row < p.n_valid ? tile * 128 + row : -1;
      else orow = row < p.rows_per_tile ? p.perm_q[(size_t)bh * p.C * p.c + (size_t)a * p.c + sub_tile * 128 + row]
                                        : -1;
      constexpr int OH = D / 2;
      __nv_bfloat16* dst = p.O + ((size_t)bh * p.N_alloc + (orow < 0 ? 0 : orow)) * D + g * OH;
#pragma unroll
      for (int c0 = 0; c0 < OH; c0 += 32) {
        uint32_t o0[32], o1[32];
        // an accumulator whose group had no block was never written
        if (jl0 >= 0) CA_TMEM_LD32(lane_addr + Cfg::kOCol + (uint32_t)(g * OH + c0), o0);
        if (jl1 >= 0) CA_TMEM_LD32(lane_addr + Cfg::kOCol + (uint32_t)(D + g * OH + c0), o1);
        tmem_wait_ld();
        if (orow >= 0) {
          uint4 w[4];
          uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            float x0 = 0.f, x1 = 0.f;
            if (jl0 >= 0) { x0 = __uint_as_float(o0[2 * q]) * w0; x1 = __uint_as_float(o0[2 * q + 1]) * w0; }
            if (jl1 >= 0) { x0 = fmaf(__uint_as_float(o1[2 * q]), w1, x0); x1 = fmaf(__uint_as_float(o1[2 * q + 1]), w1, x1); }
            wp[q] = pack_bf16(x0, x1);
          }
          uint4* gp = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
          for (int q = 0; q < 4; ++q) gp[q] = w[q];
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
// 3-D bf16 map over [BH][N_alloc][D] exposing only rows < n_valid of each head.
bool make_map_3d(CUtensorMap* m, const void* base, int BH, int N_alloc, int n_valid, int D, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)n_valid, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)N_alloc * D * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int KB>
cudaError_t launch_tc(const CUtensorMap maps[7], const TcParams& p, dim3 grid, cudaStream_t st) {
  using Cfg = TcCfg<D, KB>;
  cudaError_t e = cudaFuncSetAttribute(tc_attend_kernel<D, KB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg::kSmem);
  if (e != cudaSuccess) return e;
  tc_attend_kernel<D, KB><<<grid, Cfg::kThreads, Cfg::kSmem, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4],
                                                                   maps[5], maps[6], p);
  return cudaGetLastError();
}

// Key-block width: 128 keys, or 64 when the cluster size is 64.
int key_block(int D, int c) { return c >= 128 ? 128 : 64; (void)D; }

cudaError_t dispatch(int D, int KB, const CUtensorMap maps[7], const TcParams& p, dim3 grid, cudaStream_t st) {
  if (D == 64) return KB == 128 ? launch_tc<64, 128>(maps, p, grid, st) : launch_tc<64, 64>(maps, p, grid, st);
  return KB == 128 ? launch_tc<128, 128>(maps, p, grid, st) : launch_tc<128, 64>(maps, p, grid, st);
}

}  // namespace

cudaError_t launch_attend_tc(const ca_shape* s, const ca_clusters* cl, const ca_routes* rt, int compensate,
                             void* O, const AttendWs& L, char* ws, cudaStream_t st) {
  const int BH = s->B * s->H, D = s->d, c = s->c, C = L.C;
  const int KB = key_block(D, c);
  const uint64_t slots = (uint64_t)BH * C * c;
  CUtensorMap maps[7];
  bool ok = make_map_2d(&maps[0], ws + L.qp, slots, D, 128) && make_map_2d(&maps[1], ws + L.kp, slots, D, KB) &&
            make_map_2d(&maps[2], ws + L.vp, slots, D, KB) &&
            make_map_2d(&maps[3], ws + L.kbar_hi, (uint64_t)BH * L.Cpad, D, KB) &&
            make_map_2d(&maps[4], ws + L.kbar_lo, (uint64_t)BH * L.Cpad, D, KB) &&
            make_map_2d(&maps[5], ws + L.vbar_hi, (uint64_t)BH * L.Cpad, D, KB) &&
            make_map_2d(&maps[6], ws + L.vbar_lo, (uint64_t)BH * L.Cpad, D, KB);
  if (!ok) return cudaErrorInvalidValue;
  TcParams p;
  p.C = C; p.c = c; p.k = rt->k; p.Cpad = L.Cpad; p.n_valid = s->n_valid; p.N_alloc = s->N_alloc;
  p.tiles_per_cluster = c >= 128 ? c / 128 : 1;
  p.rows_per_tile = c >= 128 ? 128 : c;
  p.compensate = compensate;
  p.dense = 0;
  p.dense_key_blocks = 0;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  p.perm_q = cl->perm_q; p.count_k = cl->count_k; p.kept_idx = rt->kept_idx; p.kept_bits = rt->kept_bits;
  p.kept_count = rt->kept_count;
  p.logcnt = reinterpret_cast<const float*>(ws + L.logcnt);
  p.O = static_cast<__nv_bfloat16*>(O);
  p.wait_limit = wait_limit();
  const dim3 grid(C * p.tiles_per_cluster, BH);
  return dispatch(D, KB, maps, p, grid, st);
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

cudaError_t launch_dense_tc(const void* Q, const void* K, const void* V, const ca_shape* s, void* O,
                            cudaStream_t st) {
  const int BH = s->B * s->H, D = s->d;
  const int KB = key_block(D, 128);
  CUtensorMap maps[7];
  bool ok = make_map_3d(&maps[0], Q, BH, s->N_alloc, s->n_valid, D, 128) &&
            make_map_3d(&maps[1], K, BH, s->N_alloc, s->n_valid, D, KB) &&
            make_map_3d(&maps[2], V, BH, s->N_alloc, s->n_valid, D, KB);
  if (!ok) return cudaErrorInvalidValue;
  maps[3] = maps[1]; maps[4] = maps[1]; maps[5] = maps[2]; maps[6] = maps[2];
  TcParams p{};
  p.n_valid = s->n_valid; p.N_alloc = s->N_alloc;
  p.tiles_per_cluster = 1; p.rows_per_tile = 128;
  p.compensate = 0; p.dense = 1;
  p.dense_key_blocks = (s->n_valid + KB - 1) / KB;
  p.c = KB;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  p.O = static_cast<__nv_bfloat16*>(O);
  p.wait_limit = wait_limit();
  const dim3 grid((s->n_valid + 127) / 128, BH);
  return dispatch(D, KB, maps, p, grid, st);
}

}  // namespace ca
