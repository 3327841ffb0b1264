// fp32 attention on the CUDA cores (FFMA), for fp32 inputs.
//
// ClusterAttention paper, Appendix A, eq. 21-22: per query of cluster a, the
// softmax runs over every real key of the kept clusters plus, with
// compensation, one term per excluded key cluster b with logit
// q . kbar_b / sqrt(d) + ln|b| and value vbar_b. The dense form (eq. 1) runs
// over all n_valid keys.
//
// Layout: 64 query rows per block, D/16 threads per row, each thread holds 16
// interleaved dimensions (dimension e * TPR + p) of its row's q and output.
// Keys and values stream through shared memory in tiles of 32 with an
// online softmax (running max and sum) in fp32.
#include "ca_internal.cuh"

namespace ca {
namespace {

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16(v);
}

constexpr int kRows = 64;   // query rows per block
constexpr int kTile = 32;   // keys per tile

template <int D>
struct SimtState {
  static constexpr int TPR = D / 16;
  float q[16], o[16];
  float m, l;
};

template <int D>
__device__ __forceinline__ void simt_tile(SimtState<D>& st, const float* Ks, const float* Vs,
                                          const float* bias, float scale, int p) {
  constexpr int TPR = D / 16;
  float s[kTile];
  float mt = -INFINITY;
#pragma unroll
  for (int j = 0; j < kTile; ++j) {
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) part = fmaf(st.q[e], Ks[j * D + e * TPR + p], part);
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    s[j] = part * scale + bias[j];
    mt = fmaxf(mt, s[j]);
  }
  const float m_new = fmaxf(st.m, mt);
  if (m_new == -INFINITY) return;   // the whole tile is masked and nothing came before
  const float corr = (st.m == -INFINITY) ? 0.f : expf(st.m - m_new);
  st.l *= corr;
#pragma unroll
  for (int e = 0; e < 16; ++e) st.o[e] *= corr;
#pragma unroll
  for (int j = 0; j < kTile; ++j) {
    const float pj = (s[j] == -INFINITY) ? 0.f : expf(s[j] - m_new);
    st.l += pj;
#pragma unroll
    for (int e = 0; e < 16; ++e) st.o[e] = fmaf(pj, Vs[j * D + e * TPR + p], st.o[e]);
  }
  st.m = m_new;
}

// mode 0: clustered (kept blocks + optional compensation); mode 1: dense.
template <typename T, int D>
__global__ void __launch_bounds__(kRows * (D / 16)) simt_attend_kernel(
    const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V, TensorLayout TL, int n_valid,
    int c, int C, int ck, int Ck, int k, const int32_t* __restrict__ perm_q, const int32_t* __restrict__ perm_k,
    const int32_t* __restrict__ kept_idx, const uint32_t* __restrict__ kept_bits,
    const int32_t* __restrict__ kept_count, const float* __restrict__ kbar32, const float* __restrict__ vbar32, const float* __restrict__ logcnt,
    int Cpad, int compensate, int mode, float scale, T* __restrict__ O) {
  constexpr int TPR = D / 16;
  constexpr int NT = kRows * TPR;
  __shared__ float Ks[kTile * D];
  __shared__ float Vs[kTile * D];
  __shared__ float bias[kTile];
  __shared__ int krow[kTile];
  const int bh = blockIdx.y;
  const int r = threadIdx.x / TPR, p = threadIdx.x % TPR;
  const T* Qh = Q + TL.head(bh);
  const T* Kh = K + TL.head(bh);
  const T* Vh = V + TL.head(bh);
  int a = 0, row = -1;
  if (mode == 0) {
    const int per = c / kRows;
    a = blockIdx.x / per;
    const int slot = a * c + (blockIdx.x % per) * kRows + r;
    row = perm_q[(size_t)bh * C * c + slot];
  } else {
    const int rr = blockIdx.x * kRows + r;
    row = rr < n_valid ? rr : -1;
  }
  SimtState<D> st;
  st.m = -INFINITY; st.l = 0.f;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    st.q[e] = row >= 0 ? to_f(Qh[(size_t)row * TL.sn + e * TPR + p]) : 0.f;
    st.o[e] = 0.f;
  }
  auto load_rows = [&](int count_keys) {
    // krow[] and bias[] are set; stage K/V rows (zero for masked rows)
    for (int e = threadIdx.x; e < kTile * D; e += NT) {
      const int j = e / D, col = e % D;
      const int kr = krow[j];
      Ks[e] = kr >= 0 ? to_f(Kh[(size_t)kr * TL.sn + col]) : 0.f;
      Vs[e] = kr >= 0 ? to_f(Vh[(size_t)kr * TL.sn + col]) : 0.f;
    }
    (void)count_keys;
  };
  if (mode == 0) {
    const int32_t* kl = kept_idx + ((size_t)bh * C + a) * k;
    const int32_t* pk = perm_k + (size_t)bh * Ck * ck;
    // k each, or the query cluster's own count after adaptive selection
    const int kq = kept_count ? min(max(kept_count[(size_t)bh * C + a], 0), k) : k;
    for (int i = 0; i < kq; ++i) {
      const int b = kl[i];
      for (int t0 = 0; t0 < ck; t0 += kTile) {
        __syncthreads();
        if (threadIdx.x < kTile) {
          const int kr = pk[b * ck + t0 + threadIdx.x];
          krow[threadIdx.x] = kr;
          bias[threadIdx.x] = kr >= 0 ? 0.f : -INFINITY;
        }
        __syncthreads();
        load_rows(kTile);
        __syncthreads();
        simt_tile<D>(st, Ks, Vs, bias, scale, p);
      }
    }
    if (compensate) {
      const uint32_t* kb = kept_bits + ((size_t)bh * C + a) * ((Ck + 31) / 32);
      for (int b0 = 0; b0 < Ck; b0 += kTile) {
        __syncthreads();
        if (threadIdx.x < kTile) {
          const int b = b0 + threadIdx.x;
          float bs = -INFINITY;
          if (b < Ck && !((kb[b >> 5] >> (b & 31)) & 1u)) bs = logcnt[(size_t)bh * Cpad + b];
          bias[threadIdx.x] = bs;
        }
        for (int e = threadIdx.x; e < kTile * D; e += NT) {
          const int j = e / D, col = e % D, b = b0 + j;
          Ks[e] = b < Ck ? kbar32[((size_t)bh * Ck + b) * D + col] : 0.f;
          Vs[e] = b < Ck ? vbar32[((size_t)bh * Ck + b) * D + col] : 0.f;
        }
        __syncthreads();
        simt_tile<D>(st, Ks, Vs, bias, scale, p);
      }
    }
  } else {
    for (int t0 = 0; t0 < n_valid; t0 += kTile) {
      __syncthreads();
      if (threadIdx.x < kTile) {
        const int kr = t0 + threadIdx.x;
        krow[threadIdx.x] = kr < n_valid ? kr : -1;
        bias[threadIdx.x] = kr < n_valid ? 0.f : -INFINITY;
      }
      __syncthreads();
      load_rows(kTile);
      __syncthreads();
      simt_tile<D>(st, Ks, Vs, bias, scale, p);
    }
  }
  if (row >= 0) {
    const float inv = st.l > 0.f ? 1.f / st.l : 0.f;
    T* Oh = O + TL.head(bh) + (size_t)row * TL.sn;
#pragma unroll
    for (int e = 0; e < 16; ++e) Oh[e * TPR + p] = from_f<T>(st.o[e] * inv);
  }
}

template <typename T, int D>
cudaError_t run_simt(const void* Q, const void* K, const void* V, const ca_shape* s, const ca_clusters* cl,
                     const ca_routes* rt, int compensate, void* O, const AttendWs* L, char* ws, int mode,
                     cudaStream_t st) {
  const int BH = s->B * s->H, c = s->c, ck = key_c(s);
  const int C = num_q_clusters(s), Ck = num_k_clusters(s);
  const float scale = 1.0f / sqrtf((float)D);
  dim3 grid;
  if (mode == 0) grid = dim3(C * (c / kRows), BH);
  else grid = dim3((s->n_valid + kRows - 1) / kRows, BH);
  const float* kbar32 = L ? reinterpret_cast<const float*>(ws + L->kbar32) : nullptr;
  const float* vbar32 = L ? reinterpret_cast<const float*>(ws + L->vbar32) : nullptr;
  const float* logcnt = L ? reinterpret_cast<const float*>(ws + L->logcnt) : nullptr;
  simt_attend_kernel<T, D><<<grid, kRows * (D / 16), 0, st>>>(
      (const T*)Q, (const T*)K, (const T*)V, tensor_layout(s), s->n_valid, c, C, ck, Ck, rt ? rt->k : 0,
      cl ? cl->perm_q : nullptr, cl ? cl->perm_k : nullptr, rt ? rt->kept_idx : nullptr,
      rt ? rt->kept_bits : nullptr, rt ? rt->kept_count : nullptr, kbar32, vbar32, logcnt, L ? L->Cpad : 0, compensate, mode, scale,
      (T*)O);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_simt(const void* Q, const void* K, const void* V, const ca_shape* s,
                               const ca_clusters* cl, const ca_routes* rt, int compensate, void* O,
                               const AttendWs& L, char* ws, cudaStream_t st) {
  if (s->dtype == CA_FP32) {
    if (s->d == 64) return run_simt<float, 64>(Q, K, V, s, cl, rt, compensate, O, &L, ws, 0, st);
    return run_simt<float, 128>(Q, K, V, s, cl, rt, compensate, O, &L, ws, 0, st);
  }
  if (s->d == 64) return run_simt<__nv_bfloat16, 64>(Q, K, V, s, cl, rt, compensate, O, &L, ws, 0, st);
  return run_simt<__nv_bfloat16, 128>(Q, K, V, s, cl, rt, compensate, O, &L, ws, 0, st);
}

cudaError_t launch_dense_simt(const void* Q, const void* K, const void* V, const ca_shape* s, void* O,
                              cudaStream_t st) {
  if (s->dtype == CA_FP32) {
    if (s->d == 64) return run_simt<float, 64>(Q, K, V, s, nullptr, nullptr, 0, O, nullptr, nullptr, 1, st);
    return run_simt<float, 128>(Q, K, V, s, nullptr, nullptr, 0, O, nullptr, nullptr, 1, st);
  }
  if (s->d == 64)
    return run_simt<__nv_bfloat16, 64>(Q, K, V, s, nullptr, nullptr, 0, O, nullptr, nullptr, 1, st);
  return run_simt<__nv_bfloat16, 128>(Q, K, V, s, nullptr, nullptr, 0, O, nullptr, nullptr, 1, st);
}

}  // namespace ca
