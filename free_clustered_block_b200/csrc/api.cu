// libca C ABI: validation, workspace layout, and launch sequencing.
// Every check runs on the host before the first launch, so a call that
// returns an error has launched nothing.
#include <cstring>
#include <cstdio>

#include "ca_internal.cuh"

namespace ca {
size_t route_smem_bytes(int C, int D);
}  // namespace ca

using namespace ca;

namespace {

constexpr int kMaxRouteC = 8192;
// Longest accepted limit of a bounded device-side wait.
constexpr uint64_t kMaxWaitLimitNs = 10000000000ull;   // 10 s

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ca_status check_shape(const ca_shape* s) {
  if (!s) return CA_ERR_INVALID_ARG;
  if (s->B < 1 || s->H < 1 || s->n_valid < 1 || s->N_alloc < s->n_valid) return CA_ERR_INVALID_ARG;
  if (s->dtype != CA_BF16 && s->dtype != CA_FP32) return CA_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return CA_ERR_UNSUPPORTED;
  if (s->c != 64 && s->c != 128 && s->c != 256) return CA_ERR_UNSUPPORTED;
  if (s->c_k != 0 && s->c_k != 64 && s->c_k != 128 && s->c_k != 256) return CA_ERR_UNSUPPORTED;
  // every per-head index fits in int32; whole tensors fit in size_t
  const long long C = ((long long)s->n_valid + s->c - 1) / s->c;
  const long long ck = s->c_k ? s->c_k : s->c;
  const long long Ck = ((long long)s->n_valid + ck - 1) / ck;
  if ((long long)s->N_alloc > (1ll << 30) || C * s->c > (1ll << 30) || Ck * ck > (1ll << 30))
    return CA_ERR_UNSUPPORTED;
  if ((long long)s->B * s->H > 65535) return CA_ERR_UNSUPPORTED;   // grid.y
  if (s->layout != CA_LAYOUT_BHND && s->layout != CA_LAYOUT_BNHD) return CA_ERR_INVALID_ARG;
  if (s->layout == CA_LAYOUT_BHND && s->H_total != 0 && s->H_total != s->H) return CA_ERR_INVALID_ARG;
  if (s->layout == CA_LAYOUT_BNHD && s->H_total != 0 && s->H_total < s->H) return CA_ERR_INVALID_ARG;
  if (s->layout == CA_LAYOUT_BNHD && (long long)(s->H_total ? s->H_total : s->H) * s->d * 4 > (1ll << 31))
    return CA_ERR_UNSUPPORTED;
  return CA_OK;
}

bool plan_for(const ca_shape* s, TreePlan* plan) { return host_plan(s->n_valid, s->c, plan); }
bool plan_for_keys(const ca_shape* s, TreePlan* plan) { return host_plan(s->n_valid, key_c(s), plan); }

size_t dir_smem(int d, int a) {
  // one warp's share of the per-node kernel (fp32 sample rows, the larger case) plus M
  const size_t m_cap = (size_t)a * d;
  return (size_t)d * d * 8 + m_cap * (d + 1) * 4 + (2 * d + 2 * m_cap) * 8 + m_cap * 4;
}

ca_status check_params(const ca_shape* s, const ca_cluster_params* p) {
  if (!p) return CA_OK;
  if (p->power_iters < 0 || p->power_iters > 1000 || p->sample_factor < 0) return CA_ERR_INVALID_ARG;
  const int a = p->sample_factor > 0 ? p->sample_factor : 1;
  if (dir_smem(s->d, a) > 227 * 1024) return CA_ERR_UNSUPPORTED;
  if (p->transform != 0 && p->transform != 1) return CA_ERR_INVALID_ARG;
  if (p->query_form != 0 && p->query_form != 1) return CA_ERR_INVALID_ARG;
  if (p->method < 0 || p->method > 2) return CA_ERR_INVALID_ARG;
  if (p->method == 2 && a != 1) return CA_ERR_UNSUPPORTED;
  if (p->head_base < 0) return CA_ERR_INVALID_ARG;
  return CA_OK;
}

ca_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return CA_OK;
  fprintf(stderr, "libca: CUDA error %s\n", cudaGetErrorString(e));
  return CA_ERR_CUDA;
}

// Layout of ca_forward's workspace: clusters, routes, then the cluster and
// attention workspaces (which are used one after the other and may overlap).
struct ForwardWs {
  size_t perm_q, perm_k, count_q, count_k, qbar, kbar, kept_idx, kept_bits, scratch, total;
  size_t cluster_bytes, attend_bytes;
};

bool forward_layout(const ca_shape* s, int k, ForwardWs* f) {
  TreePlan plan, plan_k;
  if (!plan_for(s, &plan) || !plan_for_keys(s, &plan_k)) return false;
  ClusterWs cw;
  AttendWs aw;
  cluster_ws_layout(s, plan, plan_k, &cw);
  attend_ws_layout(s, &aw);
  const size_t BH = (size_t)s->B * s->H, C = plan.C, c = s->c, d = s->d;
  const size_t Ck = plan_k.C, ck = key_c(s);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = align_up(o + bytes); return r; };
  f->perm_q = take(BH * C * c * 4);
  f->perm_k = take(BH * Ck * ck * 4);
  f->count_q = take(BH * C * 4);
  f->count_k = take(BH * Ck * 4);
  f->qbar = take(BH * C * d * 8);
  f->kbar = take(BH * Ck * d * 8);
  f->kept_idx = take(BH * C * (size_t)k * 4);
  f->kept_bits = take(BH * C * ((Ck + 31) / 32) * 4);
  f->cluster_bytes = cw.total;
  f->attend_bytes = aw.total;
  f->scratch = take(cw.total > aw.total ? cw.total : aw.total);
  f->total = o;
  return true;
}

}  // namespace

extern "C" {

int ca_num_clusters(const ca_shape* s) {
  if (check_shape(s) != CA_OK) return -1;
  return num_q_clusters(s);
}

int ca_num_key_clusters(const ca_shape* s) {
  if (check_shape(s) != CA_OK) return -1;
  return num_k_clusters(s);
}

ca_status ca_check_shape(const ca_shape* s) { return check_shape(s); }

size_t ca_cluster_workspace_bytes(const ca_shape* s) {
  if (check_shape(s) != CA_OK) return 0;
  TreePlan plan, plan_k;
  if (!plan_for(s, &plan) || !plan_for_keys(s, &plan_k)) return 0;
  ClusterWs w;
  cluster_ws_layout(s, plan, plan_k, &w);
  return w.total;
}

size_t ca_attend_workspace_bytes(const ca_shape* s) {
  if (check_shape(s) != CA_OK) return 0;
  AttendWs w;
  attend_ws_layout(s, &w);
  return w.total;
}

size_t ca_dense_workspace_bytes(const ca_shape* s) {
  (void)s;
  return 0;
}

size_t ca_forward_workspace_bytes(const ca_shape* s, int k) {
  if (check_shape(s) != CA_OK) return 0;
  if (k < 1 || k > num_k_clusters(s)) return 0;
  ForwardWs f;
  if (!forward_layout(s, k, &f)) return 0;
  return f.total;
}

ca_status ca_cluster(const void* Q, const void* K, const ca_shape* s, const ca_cluster_params* params,
                     const ca_clusters* out, void* workspace, size_t workspace_bytes, void* stream) {
  ca_status st = check_shape(s);
  if (st != CA_OK) return st;
  if (!Q || !K || !out || !out->perm_q || !out->perm_k || !out->count_q || !out->count_k || !out->qbar ||
      !out->kbar)
    return CA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K)) return CA_ERR_INVALID_ARG;
  if ((st = check_params(s, params)) != CA_OK) return st;
  TreePlan plan, plan_k;
  if (!plan_for(s, &plan) || !plan_for_keys(s, &plan_k)) return CA_ERR_UNSUPPORTED;
  ClusterWs L;
  cluster_ws_layout(s, plan, plan_k, &L);
  if (workspace_bytes < L.total) return CA_ERR_WORKSPACE;
  if (!workspace) return CA_ERR_INVALID_ARG;
  ca_cluster_params p = {8, 1, 1, 0, 0ull, 0, 0};
  if (params) p = *params;
  return cuda_status(launch_cluster(Q, K, s, &p, out, plan, plan_k, L, static_cast<char*>(workspace),
                                    static_cast<cudaStream_t>(stream)));
}

ca_status ca_route(const ca_shape* s, const ca_clusters* cen, const ca_routes* out, void* stream) {
  ca_status st = check_shape(s);
  if (st != CA_OK) return st;
  if (!cen || !cen->qbar || !cen->kbar || !out || !out->kept_idx || !out->kept_bits) return CA_ERR_INVALID_ARG;
  if (!aligned16(cen->qbar) || !aligned16(cen->kbar)) return CA_ERR_INVALID_ARG;
  const int C = num_q_clusters(s), Ck = num_k_clusters(s);
  if (out->k < 1 || out->k > Ck) return CA_ERR_INVALID_ARG;
  if (C > kMaxRouteC || Ck > kMaxRouteC) return CA_ERR_UNSUPPORTED;
  return cuda_status(launch_route(s, C, Ck, cen->qbar, cen->kbar, out->k, out->kept_idx, out->kept_bits,
                                  out->kept_count, static_cast<cudaStream_t>(stream)));
}

ca_status ca_route_adaptive(const ca_shape* s, const ca_clusters* cen, double recall, int min_count,
                            const ca_routes* out, void* stream) {
  ca_status st = check_shape(s);
  if (st != CA_OK) return st;
  if (!cen || !cen->qbar || !cen->kbar || !cen->count_k || !out || !out->kept_idx || !out->kept_bits ||
      !out->kept_count)
    return CA_ERR_INVALID_ARG;
  if (!aligned16(cen->qbar) || !aligned16(cen->kbar)) return CA_ERR_INVALID_ARG;
  if (!(recall >= 0.0 && recall <= 1.0) || min_count < 1) return CA_ERR_INVALID_ARG;
  const int C = num_q_clusters(s), Ck = num_k_clusters(s);
  if (out->k < 1 || out->k > Ck) return CA_ERR_INVALID_ARG;
  if (C > kMaxRouteC || Ck > kMaxRouteC) return CA_ERR_UNSUPPORTED;
  return cuda_status(launch_route_adaptive(s, C, Ck, cen->qbar, cen->kbar, cen->count_k, recall, min_count, out->k,
                                           out->kept_idx, out->kept_bits, out->kept_count,
                                           static_cast<cudaStream_t>(stream)));
}

namespace {

// Checks shared by ca_attend and its two halves.
ca_status check_attend(const void* Q, const void* K, const void* V, const ca_shape* s, const ca_clusters* cl,
                       const ca_routes* rt, const void* O, size_t workspace_bytes, const void* workspace,
                       AttendWs* L) {
  ca_status st = check_shape(s);
  if (st != CA_OK) return st;
  if (!Q || !K || !V || !cl || !cl->perm_q || !cl->perm_k || !cl->count_k || !cl->kbar) return CA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V)) return CA_ERR_INVALID_ARG;
  if (rt) {
    if (!O || !rt->kept_idx || !rt->kept_bits || !aligned16(O)) return CA_ERR_INVALID_ARG;
    if (rt->k < 1 || rt->k > num_k_clusters(s)) return CA_ERR_INVALID_ARG;
  }
  attend_ws_layout(s, L);
  if (workspace_bytes < L->total) return CA_ERR_WORKSPACE;
  if (!workspace) return CA_ERR_INVALID_ARG;
  return CA_OK;
}

cudaError_t attend_blocks(const void* Q, const void* K, const void* V, const ca_shape* s, const ca_clusters* cl,
                          const ca_routes* rt, int compensate, void* O, const AttendWs& L, char* ws,
                          cudaStream_t cs) {
  cudaError_t e = (s->dtype == CA_BF16) ? launch_attend_tc(s, cl, rt, compensate, O, L, ws, cs)
                                        : launch_attend_simt(Q, K, V, s, cl, rt, compensate, O, L, ws, cs);
  if (e == cudaSuccess) e = launch_zero_pad_rows(O, s, cs);
  return e;
}

}  // namespace

ca_status ca_attend(const void* Q, const void* K, const void* V, const ca_shape* s, const ca_clusters* cl,
                    const ca_routes* rt, int compensate, void* O, void* workspace, size_t workspace_bytes,
                    void* stream) {
  if (!rt) return CA_ERR_INVALID_ARG;
  AttendWs L;
  ca_status st = check_attend(Q, K, V, s, cl, rt, O, workspace_bytes, workspace, &L);
  if (st != CA_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  cudaError_t e = launch_attend_prep(Q, K, V, s, cl, L, ws, cs);
  if (e == cudaSuccess) e = attend_blocks(Q, K, V, s, cl, rt, compensate, O, L, ws, cs);
  return cuda_status(e);
}

ca_status ca_attend_prepare(const void* Q, const void* K, const void* V, const ca_shape* s,
                            const ca_clusters* cl, void* workspace, size_t workspace_bytes, void* stream) {
  AttendWs L;
  ca_status st = check_attend(Q, K, V, s, cl, nullptr, nullptr, workspace_bytes, workspace, &L);
  if (st != CA_OK) return st;
  return cuda_status(launch_attend_prep(Q, K, V, s, cl, L, static_cast<char*>(workspace),
                                        static_cast<cudaStream_t>(stream)));
}

ca_status ca_attend_prepared(const void* Q, const void* K, const void* V, const ca_shape* s,
                             const ca_clusters* cl, const ca_routes* rt, int compensate, void* O,
                             void* workspace, size_t workspace_bytes, void* stream) {
  if (!rt) return CA_ERR_INVALID_ARG;
  AttendWs L;
  ca_status st = check_attend(Q, K, V, s, cl, rt, O, workspace_bytes, workspace, &L);
  if (st != CA_OK) return st;
  return cuda_status(attend_blocks(Q, K, V, s, cl, rt, compensate, O, L, static_cast<char*>(workspace),
                                   static_cast<cudaStream_t>(stream)));
}

ca_status ca_dense_attend(const void* Q, const void* K, const void* V, const ca_shape* s, void* O,
                          void* workspace, size_t workspace_bytes, void* stream) {
  (void)workspace; (void)workspace_bytes;
  ca_status st = check_shape(s);
  if (st != CA_OK) return st;
  if (!Q || !K || !V || !O) return CA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return CA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e = (s->dtype == CA_BF16) ? launch_dense_tc(Q, K, V, s, O, cs)
                                        : launch_dense_simt(Q, K, V, s, O, cs);
  if (e == cudaSuccess) e = launch_zero_pad_rows(O, s, cs);
  return cuda_status(e);
}

ca_status ca_forward(const void* Q, const void* K, const void* V, const ca_shape* s,
                     const ca_cluster_params* params, int k, int compensate, void* O, void* workspace,
                     size_t workspace_bytes, void* stream) {
  ca_status st = check_shape(s);
  if (st != CA_OK) return st;
  if (!Q || !K || !V || !O) return CA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return CA_ERR_INVALID_ARG;
  if ((st = check_params(s, params)) != CA_OK) return st;
  if (k < 1 || k > num_k_clusters(s)) return CA_ERR_INVALID_ARG;
  if (num_q_clusters(s) > kMaxRouteC || num_k_clusters(s) > kMaxRouteC) return CA_ERR_UNSUPPORTED;
  ForwardWs f;
  if (!forward_layout(s, k, &f)) return CA_ERR_UNSUPPORTED;
  if (workspace_bytes < f.total) return CA_ERR_WORKSPACE;
  if (!workspace) return CA_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  ca_clusters cl;
  cl.perm_q = reinterpret_cast<int32_t*>(ws + f.perm_q);
  cl.perm_k = reinterpret_cast<int32_t*>(ws + f.perm_k);
  cl.count_q = reinterpret_cast<int32_t*>(ws + f.count_q);
  cl.count_k = reinterpret_cast<int32_t*>(ws + f.count_k);
  cl.qbar = reinterpret_cast<double*>(ws + f.qbar);
  cl.kbar = reinterpret_cast<double*>(ws + f.kbar);
  ca_routes rt;
  rt.k = k;
  rt.kept_count = nullptr;
  rt.kept_idx = reinterpret_cast<int32_t*>(ws + f.kept_idx);
  rt.kept_bits = reinterpret_cast<uint32_t*>(ws + f.kept_bits);
  st = ca_cluster(Q, K, s, params, &cl, ws + f.scratch, f.cluster_bytes, stream);
  if (st != CA_OK) return st;
  st = ca_route(s, &cl, &rt, stream);
  if (st != CA_OK) return st;
  return ca_attend(Q, K, V, s, &cl, &rt, compensate, O, ws + f.scratch, f.attend_bytes, stream);
}

}  // extern "C"

namespace {

// ca_forward_host pipelines groups of heads: the host-to-device copies of one
// group overlap the forward of the previous one and the device-to-host copy
// of the one before. Groups are contiguous ranges of the flattened heads,
// sizes differing by at most one (the first groups take one more).
constexpr int kHostGroups = 4;

int host_groups(const ca_shape* s) {
  // a group of heads is a contiguous byte range only in the [B][H][N][d] layout
  if (s->layout != CA_LAYOUT_BHND) return 1;
  const int BH = s->B * s->H;
  return BH < kHostGroups ? BH : kHostGroups;
}

// Shape of group g: B = 1, H = the group's head count; first flattened head in
// *first. A single group is the whole shape.
ca_shape group_shape(const ca_shape* s, int g, int G, int* first) {
  if (G == 1) { *first = 0; return *s; }
  const int BH = s->B * s->H, base = BH / G, extra = BH % G;
  *first = g * base + (g < extra ? g : extra);
  ca_shape gs = *s;
  gs.B = 1;
  gs.H = base + (g < extra ? 1 : 0);
  return gs;
}

}  // namespace

extern "C" {

size_t ca_forward_host_workspace_bytes(const ca_shape* s, int k) {
  if (check_shape(s) != CA_OK) return 0;
  if (!layout_contiguous(s)) return 0;   // host buffers hold exactly the call's heads
  int first = 0;
  const ca_shape g0 = group_shape(s, 0, host_groups(s), &first);   // the largest group
  const size_t base = ca_forward_workspace_bytes(&g0, k);
  if (!base) return 0;
  const size_t esz = s->dtype == CA_BF16 ? 2 : 4;
  const size_t t = (size_t)s->B * s->H * s->N_alloc * s->d * esz;
  return base + 4 * align_up(t);
}

ca_status ca_forward_host(const void* Qh, const void* Kh, const void* Vh, const ca_shape* s,
                          const ca_cluster_params* params, int k, int compensate, void* Oh, void* workspace,
                          size_t workspace_bytes, void* stream) {
  ca_status st = check_shape(s);
  if (st != CA_OK) return st;
  if (!layout_contiguous(s)) return CA_ERR_UNSUPPORTED;
  if (!Qh || !Kh || !Vh || !Oh) return CA_ERR_INVALID_ARG;
  if ((st = check_params(s, params)) != CA_OK) return st;
  const size_t need = ca_forward_host_workspace_bytes(s, k);
  if (!need) return CA_ERR_INVALID_ARG;
  if (workspace_bytes < need) return CA_ERR_WORKSPACE;
  if (!workspace) return CA_ERR_INVALID_ARG;
  const int G = host_groups(s);
  const size_t esz = s->dtype == CA_BF16 ? 2 : 4;
  const size_t head_bytes = (size_t)s->N_alloc * s->d * esz;
  const size_t t = (size_t)s->B * s->H * head_bytes;
  char* ws = static_cast<char*>(workspace);
  int first = 0;
  const ca_shape g0 = group_shape(s, 0, G, &first);
  const size_t base = ca_forward_workspace_bytes(&g0, k);
  char* dQ = ws + base;
  char* dK = dQ + align_up(t);
  char* dV = dK + align_up(t);
  char* dO = dV + align_up(t);
  ca_cluster_params p = {8, 1, 1, 0, 0ull, 0, 0};
  if (params) p = *params;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // helper streams for the two copy directions, and their events
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_in[kHostGroups] = {}, ev_out[kHostGroups] = {};
  cudaError_t e = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking);
  for (int g = 0; g < G && e == cudaSuccess; ++g) {
    e = cudaEventCreateWithFlags(&ev_in[g], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_out[g], cudaEventDisableTiming);
  }
  // the inputs must not be overwritten before earlier work on `stream` is done with them
  cudaEvent_t ev_start = nullptr;
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventRecord(ev_start, cs);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, ev_start, 0);
  for (int g = 0; g < G && e == cudaSuccess; ++g) {
    int b0 = 0;
    const ca_shape gs = group_shape(s, g, G, &b0);
    const size_t off = (size_t)b0 * head_bytes, bytes = G == 1 ? t : (size_t)gs.H * head_bytes;
    e = cudaMemcpyAsync(dQ + off, static_cast<const char*>(Qh) + off, bytes, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(dK + off, static_cast<const char*>(Kh) + off, bytes, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(dV + off, static_cast<const char*>(Vh) + off, bytes, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess) e = cudaEventRecord(ev_in[g], s_in);
  }
  for (int g = 0; g < G && e == cudaSuccess && st == CA_OK; ++g) {
    int b0 = 0;
    const ca_shape gs = group_shape(s, g, G, &b0);
    const size_t off = (size_t)b0 * head_bytes, bytes = G == 1 ? t : (size_t)gs.H * head_bytes;
    e = cudaStreamWaitEvent(cs, ev_in[g], 0);
    if (e != cudaSuccess) break;
    ca_cluster_params pg = p;
    pg.head_base = p.head_base + b0;
    st = ca_forward(dQ + off, dK + off, dV + off, &gs, &pg, k, compensate, dO + off, ws, base, stream);
    if (st != CA_OK) break;
    e = cudaEventRecord(ev_out[g], cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_out[g], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<char*>(Oh) + off, dO + off, bytes, cudaMemcpyDeviceToHost, s_out);
  }
  // wait for everything issued on the three streams, then release the helpers
  if (s_in) { const cudaError_t e2 = cudaStreamSynchronize(s_in); if (e == cudaSuccess) e = e2; }
  { const cudaError_t e2 = cudaStreamSynchronize(cs); if (e == cudaSuccess) e = e2; }
  if (s_out) { const cudaError_t e2 = cudaStreamSynchronize(s_out); if (e == cudaSuccess) e = e2; }
  for (int g = 0; g < G; ++g) {
    if (ev_in[g]) cudaEventDestroy(ev_in[g]);
    if (ev_out[g]) cudaEventDestroy(ev_out[g]);
  }
  if (ev_start) cudaEventDestroy(ev_start);
  if (s_in) cudaStreamDestroy(s_in);
  if (s_out) cudaStreamDestroy(s_out);
  if (st != CA_OK) return st;
  return cuda_status(e);
}

ca_status ca_get_device_error(void* stream) {
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return cuda_status(e);
  unsigned word = 0;
  e = device_error_read_clear(&word, cs);
  if (e != cudaSuccess) return cuda_status(e);
  return word ? static_cast<ca_status>(word) : CA_OK;
}

ca_status ca_set_wait_limit(uint64_t limit_ns) {
  if (limit_ns > kMaxWaitLimitNs) return CA_ERR_INVALID_ARG;
  set_wait_limit(limit_ns);
  return CA_OK;
}

ca_status ca_check_bounded_wait(uint64_t limit_ns, int arrive, void* stream) {
  if (limit_ns == 0 || limit_ns > kMaxWaitLimitNs) return CA_ERR_INVALID_ARG;
  return cuda_status(launch_bounded_wait_check(limit_ns, arrive ? 1 : 0, static_cast<cudaStream_t>(stream)));
}

ca_status ca_check_exp2_poly(const float* x, float* y, int n, void* stream) {
  if (n < 0) return CA_ERR_INVALID_ARG;
  if (n == 0) return CA_OK;   // nothing is read or written
  if (!x || !y) return CA_ERR_INVALID_ARG;
  return cuda_status(launch_exp2_poly_check(x, y, n, static_cast<cudaStream_t>(stream)));
}

int ca_launch_count(const ca_shape* s, int stage) {
  if (check_shape(s) != CA_OK) return -1;
  const int pad = s->N_alloc > s->n_valid ? 1 : 0;
  switch (stage) {
    case 0: {
      TreePlan plan, plan_k;
      if (!plan_for(s, &plan) || !plan_for_keys(s, &plan_k)) return -1;
      // plan, colsum, syrk, metric reduce, query norms; per level: direction,
      // projection, select, partition count, partition scatter; centroids.
      // With unequal sizes each tensor walks its own tree (a plan and a
      // centroid launch each).
      if (key_c(s) == s->c) return plan.levels > 0 ? 5 + 5 * plan.levels + 1 : 1;
      const bool any = plan.levels > 0 || plan_k.levels > 0;
      return (any ? 2 + 4 : 0) + 5 * (plan.levels + plan_k.levels) + 2;
    }
    case 1: return 1;
    case 2: return (s->dtype == CA_BF16 ? 2 : 1) + 1 + pad;   // prep (+ permute), attention, pad rows
    case 3: return 1 + pad;
  }
  return -1;
}

const char* ca_status_string(ca_status s) {
  switch (s) {
    case CA_OK: return "CA_OK";
    case CA_ERR_INVALID_ARG: return "CA_ERR_INVALID_ARG";
    case CA_ERR_UNSUPPORTED: return "CA_ERR_UNSUPPORTED";
    case CA_ERR_WORKSPACE: return "CA_ERR_WORKSPACE";
    case CA_ERR_CUDA: return "CA_ERR_CUDA";
    case CA_ERR_TIMEOUT: return "CA_ERR_TIMEOUT";
  }
  return "CA_ERR_UNKNOWN";
}

const char* ca_version(void) { return "libca 0.1 (sm_100a)"; }

}  // extern "C"
