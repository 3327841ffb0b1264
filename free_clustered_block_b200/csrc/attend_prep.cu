// Attention preparation: value centroids, compensation terms, and the
// cluster-ordered copies of Q, K and V that the tensor-core kernel tiles.
//
// ClusterAttention paper, Appendix A, eq. 21-22: every excluded key cluster b
// enters a query's softmax as one term with logit q . kbar_b / sqrt(d) + ln|b|
// and value vbar_b, the mean value of its |b| real members.
//
// Centroids are fp64 from clustering. For the bf16 tensor-core path each
// fp64 centroid is split into bf16 hi + lo parts (x ~ hi + lo, ~16 significant
// bits) so that two bf16 products carry it into the fp32 accumulator.
#include "ca_internal.cuh"

namespace ca {
namespace {

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// One block per key cluster: vbar (fp64 mean of the members' values), and the
// fp32 / bf16 hi-lo forms of kbar and vbar; log count. The hi-lo forms are
// laid out in blocks of 64 centroids as the tensor-core kernel loads them:
// block cb holds the hi parts of centroids 64 cb .. 64 cb + 63 in rows 0-63
// and their lo parts in rows 64-127 ([BH][Cpad / 64][128][D]).
template <typename T, int D>
__global__ void __launch_bounds__(256) centroid_prep_kernel(
    const T* __restrict__ V, TensorLayout TL, int c, int C, int Cpad, const int32_t* __restrict__ perm_k,
    const int32_t* __restrict__ count_k, const double* __restrict__ kbar, float* __restrict__ kbar32,
    float* __restrict__ vbar32, __nv_bfloat16* __restrict__ kbar_hl, __nv_bfloat16* __restrict__ vbar_hl,
    float* __restrict__ logcnt) {
  constexpr int RG = 256 / D;
  const int b = blockIdx.x, bh = blockIdx.y;
  const int col = threadIdx.x % D, rg = threadIdx.x / D;
  const size_t o_hi = (((size_t)bh * (Cpad / 64) + b / 64) * 128 + (b % 64)) * D + col;
  const size_t o_lo = o_hi + (size_t)64 * D;
  if (b >= C) {   // padding centroids of the tensor-core tiles
    if (rg == 0) {
      const __nv_bfloat16 z = __float2bfloat16(0.f);
      kbar_hl[o_hi] = z; kbar_hl[o_lo] = z; vbar_hl[o_hi] = z; vbar_hl[o_lo] = z;
      if (col == 0) logcnt[(size_t)bh * Cpad + b] = -INFINITY;
    }
    return;
  }
  const int cnt = count_k[(size_t)bh * C + b];
  const int32_t* mem = perm_k + (size_t)bh * C * c + (size_t)b * c;
  const T* Vh = V + TL.head(bh);
  // members rg, rg + RG, ... summed in that order, four row loads in flight
  double s = 0.0;
  int j = rg;
  for (; j + 3 * RG < cnt; j += 4 * RG) {
    const int r0 = mem[j], r1 = mem[j + RG], r2 = mem[j + 2 * RG], r3 = mem[j + 3 * RG];
    const T x0 = Vh[(size_t)r0 * TL.sn + col], x1 = Vh[(size_t)r1 * TL.sn + col];
    const T x2 = Vh[(size_t)r2 * TL.sn + col], x3 = Vh[(size_t)r3 * TL.sn + col];
    s += (double)to_f(x0);
    s += (double)to_f(x1);
    s += (double)to_f(x2);
    s += (double)to_f(x3);
  }
  for (; j < cnt; j += RG) s += (double)to_f(Vh[(size_t)mem[j] * TL.sn + col]);
  __shared__ double red[256];
  red[threadIdx.x] = s;
  __syncthreads();
  if (rg == 0) {
    double t = 0.0;
    for (int g = 0; g < RG; ++g) t += red[g * D + col];
    const double vb = t / (double)cnt;
    const double kb = kbar[((size_t)bh * C + b) * D + col];
    const size_t o32 = ((size_t)bh * C + b) * D + col;
    vbar32[o32] = (float)vb;
    kbar32[o32] = (float)kb;
    const __nv_bfloat16 khi = __double2bfloat16(kb);
    const __nv_bfloat16 vhi = __double2bfloat16(vb);
    kbar_hl[o_hi] = khi; kbar_hl[o_lo] = __double2bfloat16(kb - (double)__bfloat162float(khi));
    vbar_hl[o_hi] = vhi; vbar_hl[o_lo] = __double2bfloat16(vb - (double)__bfloat162float(vhi));
    if (col == 0) logcnt[(size_t)bh * Cpad + b] = logf((float)cnt);
  }
}

// Cluster-ordered copy: dst[bh][slot] = src[bh][perm[slot]] (zero for pad
// slots). One 16-byte vector per thread; blockIdx.z selects Q / K / V. The
// queries have slots_q slots per head (query clusters of c), keys and values
// slots_k (key clusters of c_k).
template <int D>
__global__ void __launch_bounds__(256) permute_rows_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
    const __nv_bfloat16* __restrict__ V, TensorLayout TL, int slots_q, int slots_k, const int32_t* __restrict__ perm_q,
    const int32_t* __restrict__ perm_k, __nv_bfloat16* __restrict__ Qp, __nv_bfloat16* __restrict__ Kp,
    __nv_bfloat16* __restrict__ Vp) {
  constexpr int VPR = D * 2 / 16;   // 16-byte vectors per row
  const int bh = blockIdx.y, z = blockIdx.z;
  const int slots = z == 0 ? slots_q : slots_k;
  const __nv_bfloat16* src = (z == 0 ? Q : (z == 1 ? K : V)) + TL.head(bh);
  __nv_bfloat16* dst = (z == 0 ? Qp : (z == 1 ? Kp : Vp)) + (size_t)bh * slots * D;
  const int32_t* perm = (z == 0 ? perm_q : perm_k) + (size_t)bh * slots;
  const size_t e = (size_t)blockIdx.x * 256 + threadIdx.x;
  const int slot = (int)(e / VPR), v = (int)(e % VPR);
  if (slot >= slots) return;
  const int row = perm[slot];
  uint4 val = make_uint4(0, 0, 0, 0);
  if (row >= 0) val = *reinterpret_cast<const uint4*>(src + (size_t)row * TL.sn + v * 8);
  *reinterpret_cast<uint4*>(dst + (size_t)slot * D + v * 8) = val;
}

// O rows first_row .. first_row + pad_rows - 1 of head blockIdx.y (TL in
// 16-byte vectors): thread (x, y) zeroes vector x of one row.
__global__ void zero_rows_kernel(uint4* __restrict__ O, TensorLayout TL, int first_row, int pad_rows) {
  const int r = blockIdx.x * blockDim.y + threadIdx.y;
  if (r >= pad_rows) return;
  O[TL.head(blockIdx.y) + (long long)(first_row + r) * TL.sn + threadIdx.x] = make_uint4(0, 0, 0, 0);
}

}  // namespace

bool attend_ws_layout(const ca_shape* s, AttendWs* w) {
  const size_t BH = (size_t)s->B * s->H, d = s->d, c = s->c, ck = key_c(s);
  const size_t C = num_q_clusters(s), Ck = num_k_clusters(s);
  const size_t Cpad = (Ck + 127) / 128 * 128;
  w->C = (int)C; w->Ck = (int)Ck; w->Cpad = (int)Cpad;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = align_up(o + bytes); return r; };
  const bool tc = (s->dtype == CA_BF16);
  const size_t rows_q = BH * C * c * d * 2, rows_k = BH * Ck * ck * d * 2;
  w->qp = take(tc ? rows_q : 0);
  w->kp = take(tc ? rows_k : 0);
  w->vp = take(tc ? rows_k : 0);
  w->kbar_hl = take(BH * Cpad * 2 * d * 2);
  w->vbar_hl = take(BH * Cpad * 2 * d * 2);
  w->vbar32 = take(BH * Ck * d * 4);
  w->kbar32 = take(BH * Ck * d * 4);
  w->logcnt = take(BH * Cpad * 4);
  w->total = o;
  return true;
}

cudaError_t launch_attend_prep(const void* Q, const void* K, const void* V, const ca_shape* s,
                               const ca_clusters* cl, const AttendWs& L, char* ws, cudaStream_t st) {
  // key centroids: C key clusters of c = c_k slots
  const int BH = s->B * s->H, C = L.Ck, Cpad = L.Cpad, c = key_c(s);
  float* kbar32 = reinterpret_cast<float*>(ws + L.kbar32);
  float* vbar32 = reinterpret_cast<float*>(ws + L.vbar32);
  __nv_bfloat16* khl = reinterpret_cast<__nv_bfloat16*>(ws + L.kbar_hl);
  __nv_bfloat16* vhl = reinterpret_cast<__nv_bfloat16*>(ws + L.vbar_hl);
  float* logcnt = reinterpret_cast<float*>(ws + L.logcnt);
  const dim3 g(Cpad, BH);
  const TensorLayout TL = tensor_layout(s);
  if (s->dtype == CA_BF16) {
    using T = __nv_bfloat16;
    if (s->d == 64)
      centroid_prep_kernel<T, 64><<<g, 256, 0, st>>>((const T*)V, TL, c, C, Cpad, cl->perm_k,
                                                     cl->count_k, cl->kbar, kbar32, vbar32, khl, vhl, logcnt);
    else
      centroid_prep_kernel<T, 128><<<g, 256, 0, st>>>((const T*)V, TL, c, C, Cpad, cl->perm_k,
                                                      cl->count_k, cl->kbar, kbar32, vbar32, khl, vhl, logcnt);
    const int slots_q = L.C * s->c, slots_k = C * c;
    const int slots = slots_q > slots_k ? slots_q : slots_k;
    const size_t vecs = (size_t)slots * (s->d * 2 / 16);
    const dim3 gp((unsigned)((vecs + 255) / 256), BH, 3);
    T* Qp = reinterpret_cast<T*>(ws + L.qp);
    T* Kp = reinterpret_cast<T*>(ws + L.kp);
    T* Vp = reinterpret_cast<T*>(ws + L.vp);
    if (s->d == 64)
      permute_rows_kernel<64><<<gp, 256, 0, st>>>((const T*)Q, (const T*)K, (const T*)V, TL, slots_q,
                                                  slots_k, cl->perm_q, cl->perm_k, Qp, Kp, Vp);
    else
      permute_rows_kernel<128><<<gp, 256, 0, st>>>((const T*)Q, (const T*)K, (const T*)V, TL,
                                                   slots_q, slots_k, cl->perm_q, cl->perm_k, Qp, Kp, Vp);
  } else {
    using T = float;
    if (s->d == 64)
      centroid_prep_kernel<T, 64><<<g, 256, 0, st>>>((const T*)V, TL, c, C, Cpad, cl->perm_k,
                                                     cl->count_k, cl->kbar, kbar32, vbar32, khl, vhl, logcnt);
    else
      centroid_prep_kernel<T, 128><<<g, 256, 0, st>>>((const T*)V, TL, c, C, Cpad, cl->perm_k,
                                                      cl->count_k, cl->kbar, kbar32, vbar32, khl, vhl, logcnt);
  }
  return cudaGetLastError();
}

cudaError_t launch_zero_pad_rows(void* O, const ca_shape* s, cudaStream_t st) {
  if (s->N_alloc <= s->n_valid) return cudaSuccess;
  const int esz = (s->dtype == CA_BF16) ? 2 : 4;
  const int row_vecs = s->d * esz / 16;   // 8, 16 or 32
  const int BH = s->B * s->H;
  const int pad = s->N_alloc - s->n_valid;
  // the layout in 16-byte vectors (every stride is a whole number of rows of d elements)
  TensorLayout TV = tensor_layout(s);
  const long long vec = 16 / esz;
  TV.sb /= vec; TV.sh /= vec; TV.sn /= vec;
  const dim3 block(row_vecs, 256 / row_vecs);
  const dim3 grid((pad + block.y - 1) / block.y, BH);
  zero_rows_kernel<<<grid, block, 0, st>>>(reinterpret_cast<uint4*>(O), TV, s->n_valid, pad);
  return cudaGetLastError();
}

}  // namespace ca
