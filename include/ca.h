/*
 * ca.h -- C ABI of libca, the B200 (sm_100a) ClusterAttention forward path.
 *
 * The operation is the forward pass of one bidirectional attention layer as
 * described in "ClusterAttention: A training-free speedup of bidirectional
 * attention" (arXiv 2608.26965), Section 1.1 (the four steps: cluster keys
 * and queries, score and select key clusters per query cluster, attend over
 * the selected clusters, compensate the unselected ones) and Section 3.1
 * ("Overview": clustering, assignment, attention, per attention head).
 *
 * Conventions for every entry point:
 *  - Tensor pointers are DEVICE pointers owned by the caller, except where a
 *    name ends in _host. Nothing here allocates or frees device memory; work
 *    that needs scratch takes a caller-provided workspace whose size is given
 *    by the matching *_workspace_bytes() query.
 *  - Q, K, V and O share the shape's layout (ca_layout: head-major
 *    [B][H][N_alloc][d] or token-major [B][N_alloc][H_total][d]), each row of
 *    d elements contiguous, 16-byte aligned. Rows (tokens) n_valid..N_alloc-1
 *    are padding: never read as tokens; O's padding rows are written as 0.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream). Calls are asynchronous on it and never synchronise the host,
 *    except ca_get_device_error() and the _host variant.
 *  - Arguments are validated on the host before any launch; a call that
 *    returns an error status has launched nothing and written nothing.
 *  - Clustering, routing and the centroid-score arithmetic are fp64; the
 *    attention computes in fp32 (fp32 inputs) or bf16 tensor-core products
 *    with fp32 accumulation (bf16 inputs).
 */
#ifndef CA_H
#define CA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CA_OK = 0,
  CA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, k out of range, misaligned base */
  CA_ERR_UNSUPPORTED = 2,   /* valid but not built: d not in {64,128}, c not in {64,128,256} ... */
  CA_ERR_WORKSPACE = 3,     /* workspace smaller than the *_workspace_bytes() query */
  CA_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed */
  CA_ERR_TIMEOUT = 5        /* a bounded device-side wait gave up (see ca_get_device_error) */
} ca_status;

typedef enum { CA_BF16 = 0, CA_FP32 = 1 } ca_dtype;

/* Memory layout of Q, K, V and O (the same for all four):
 *  CA_LAYOUT_BHND  [B][H][N_alloc][d], each head's rows contiguous;
 *  CA_LAYOUT_BNHD  [B][N_alloc][H_total][d], the heads of one token
 *                  contiguous (the layout a fused QKV projection produces);
 *                  the call's H heads are heads 0..H-1 of the pointers, so a
 *                  slice of heads h0..h0+H-1 passes pointers offset by h0*d. */
typedef enum { CA_LAYOUT_BHND = 0, CA_LAYOUT_BNHD = 1 } ca_layout;

/* Problem shape. C = ceil(n_valid / c) query clusters and
 * C_k = ceil(n_valid / c_k) key clusters (c_k = 0 means c_k = c, so C_k = C).
 * Unequal sizes are the paper's evaluated block shape (Section 3.1,
 * "Overview": 64 queries against 128 keys per block).
 * Supported: d in {64, 128}; c and c_k in {64, 128, 256}; 1 <= n_valid <=
 * N_alloc; dtype CA_BF16 or CA_FP32; layout CA_LAYOUT_BHND or CA_LAYOUT_BNHD. */
typedef struct {
  int B, H;          /* batch, heads */
  int N_alloc;       /* rows allocated per head */
  int n_valid;       /* tokens per head (rows 0..n_valid-1) */
  int d;             /* head dimension */
  int c;             /* query cluster size (and key cluster size when c_k is 0) */
  int dtype;         /* ca_dtype of Q, K, V and O */
  int c_k;           /* key cluster size, or 0 for c */
  int layout;        /* ca_layout of Q, K, V and O */
  int H_total;       /* CA_LAYOUT_BNHD: heads per token in memory (>= H), or 0 for H;
                        CA_LAYOUT_BHND: 0 or H */
} ca_shape;

/* Clustering knobs (paper Section 3.2.1, "Basic recursive splitting" and
 * "Diagonalized recursive splitting"):
 *  power_iters   p, power-iteration steps per split (0 -> default 8);
 *  sample_factor a, sample size min(a d, |S|) per split (0 -> default 1);
 *  transform     1 = interaction-aware transforms (Section 3.2.2), the default;
 *                0 = split the raw vectors (the paper's ablation);
 *  query_form    0 = queries as R_k q / |R_k q| (eq. 16, for top-k selection),
 *                    the default; 1 = queries as R_k q (eq. 15, for adaptive
 *                    selection); ignored when transform is 0;
 *  seed          counter-based generator seed for samples and warm starts;
 *  method        0 = recursive splitting (the method), the default;
 *                1 = random clusters, the baseline of the paper's error
 *                    analysis: token i of (b, h, tensor) gets the key
 *                    SplitMix64(stream(seed, bh, tensor, 0) ^ i), and the
 *                    tokens ordered by (key, i) form the clusters, c at a
 *                    time, the remainder last (the other knobs are ignored);
 *                2 = diagonalized recursive splitting: the representations
 *                    are rotated once into the principal-component basis of
 *                    the full set (eigenvectors u_j of their covariance by
 *                    descending eigenvalue, each signed so that the
 *                    raw-space direction R u_j has its largest-magnitude
 *                    entry positive) and every set is
 *                    split on the coordinate with the highest variance over
 *                    the basic splitting's sample (lowest index on a tie);
 *                    power_iters is ignored; sample_factor must be 0 or 1
 *                    (CA_ERR_UNSUPPORTED otherwise);
 *  head_base     global index of this call's first (b, h) pair, >= 0 (0 for a
 *                whole layer): the random streams of head (b, h) are keyed by
 *                head_base + b*H + h, so a call on a slice of a layer's heads
 *                (pointers offset to the slice, H the slice's head count)
 *                reproduces exactly the clusters the whole-layer call makes
 *                for those heads. This is how one layer's heads are split
 *                across GPUs. */
typedef struct {
  int power_iters;
  int sample_factor;
  int transform;
  int query_form;
  uint64_t seed;
  int method;
  int head_base;
} ca_cluster_params;

/* Clustering result, one entry per (b, h), C = ca_num_clusters(shape) query
 * clusters of c slots and C_k = ca_num_key_clusters(shape) key clusters of
 * c_k slots:
 *  perm_q          int32 [B][H][C*c], perm_k int32 [B][H][C_k*c_k]: slot a*c+j
 *                  holds the original row of the j-th member of cluster a
 *                  (ascending rows); -1 in pad slots. Every cluster is full
 *                  except possibly the last, which holds the remainder
 *                  (Section 3.1).
 *  count_q         int32 [B][H][C], count_k int32 [B][H][C_k]: members per cluster.
 *  qbar            fp64 [B][H][C][d], kbar fp64 [B][H][C_k][d]: centroids in
 *                  the original, untransformed space (Section 3.3.1, eq. 18). */
typedef struct {
  int32_t* perm_q;
  int32_t* perm_k;
  int32_t* count_q;
  int32_t* count_k;
  double* qbar;
  double* kbar;
} ca_clusters;

/* Routing result (C query clusters, C_k key clusters):
 *  kept_idx   int32 [B][H][C][k]: the key clusters kept by each query
 *             cluster, ascending (row stride k), 1 <= k <= C_k;
 *  kept_bits  uint32 [B][H][C][ceil(C_k/32)]: the same set as a bitmask
 *             (bit b%32 of word b/32);
 *  kept_count int32 [B][H][C] or NULL: how many entries of each kept_idx row
 *             are used. NULL means every query cluster keeps exactly k (top-k
 *             selection); ca_route writes k into it when given, and
 *             ca_route_adaptive requires it (entries past the count are
 *             unspecified). */
typedef struct {
  int k;
  int32_t* kept_idx;
  uint32_t* kept_bits;
  int32_t* kept_count;
} ca_routes;

/* Number of query clusters C = ceil(n_valid / c); -1 if the shape is invalid. Host only. */
int ca_num_clusters(const ca_shape* shape);

/* Number of key clusters C_k = ceil(n_valid / c_k) (C when c_k is 0); -1 if
 * the shape is invalid. Host only. */
int ca_num_key_clusters(const ca_shape* shape);

/* Validate a shape without launching anything. Host only. */
ca_status ca_check_shape(const ca_shape* shape);

/* Workspace sizes in bytes (0 if the shape is invalid). Host only, pure. */
size_t ca_cluster_workspace_bytes(const ca_shape* shape);
size_t ca_attend_workspace_bytes(const ca_shape* shape);
size_t ca_dense_workspace_bytes(const ca_shape* shape);
size_t ca_forward_workspace_bytes(const ca_shape* shape, int k);

/*
 * ca_cluster -- cluster the queries and the keys of every head.
 * Paper Section 3.2 "Clustering": per head and separately for Q and K,
 * the metric matrices M_q = Q^T Q / n (eq. 10-12) and M_k = K_c^T K_c / n
 * (eq. 15, centred keys); keys are split in the space R_q k (eq. 14), queries
 * in R_k q / |R_k q| (eq. 16); basic recursive splitting (PDDP): per set S,
 * sample min(a d, |S|) vectors, estimate the first principal component by
 * power iteration (warm-started from the mean of the parent's estimate and a
 * random normal vector), project S, put the multiple of c closest to |S|/2
 * below the split, recurse until every set but at most one holds c vectors.
 * The metric is injected into the power iteration (Section 6.1), so no
 * eigendecomposition is run. Ties between equal projections go by row index.
 * Q, K: device, shape->dtype, in shape->layout. out: device buffers, see
 * ca_clusters. workspace: device, >= ca_cluster_workspace_bytes(shape).
 * Errors: CA_ERR_INVALID_ARG / CA_ERR_UNSUPPORTED / CA_ERR_WORKSPACE before
 * any launch; CA_ERR_CUDA if a launch fails.
 */
ca_status ca_cluster(const void* Q, const void* K, const ca_shape* shape,
                     const ca_cluster_params* params, const ca_clusters* out,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * ca_cluster_noalloc -- ca_cluster for callers that cannot allocate device
 * memory: plugins inside another framework that owns every device allocation
 * and gives no scratch buffer, and latency-critical loops that must not call
 * cudaMalloc (it can synchronise the device and can fail mid-run). The paper
 * has no counterpart; this is a deployment convenience of this library.
 * Same arguments and results as ca_cluster, without the workspace: the
 * scratch is a fixed 16 MiB array in device memory that belongs to the
 * library (every GPU on which it is loaded holds those 16 MiB until the
 * process exits). Shapes whose ca_cluster_workspace_bytes() exceeds 16 MiB
 * are rejected with CA_ERR_WORKSPACE before any launch (e.g. two
 * 65,536-token heads at d = 64 fit, eight do not). Nothing here calls
 * cudaMalloc, cudaFree or any allocating routine. The first call on a device
 * looks up the array's device address (with that device current), so make
 * that first call before any stream capture; the address is looked up again
 * when the current context is no longer the one it was found in (after
 * cudaDeviceReset, for example). All calls share the one array:
 * calls whose work overlaps on the GPU (different streams, or several host
 * threads) race on it and must be serialised by the caller.
 */
ca_status ca_cluster_noalloc(const void* Q, const void* K, const ca_shape* shape,
                             const ca_cluster_params* params, const ca_clusters* out,
                             void* stream);

/*
 * ca_route -- centroid scores and top-k selection.
 * Paper Section 3.3.1 (score s_ab = qbar_a . kbar_b, eq. 18, computed in fp64)
 * and Section 3.3.2 (keep the k best-scoring key clusters per query cluster).
 * Exact top-k; equal scores go to the lower key-cluster index.
 * centroids: device qbar/kbar (fp64) as produced by ca_cluster or supplied by
 * the caller; only qbar and kbar are read, and both must be 16-byte aligned
 * (CA_ERR_INVALID_ARG otherwise). out: device kept_idx and kept_bits;
 * out->k is k. 1 <= k <= C_k; C, C_k <= 8192.
 */
ca_status ca_route(const ca_shape* shape, const ca_clusters* centroids,
                   const ca_routes* out, void* stream);

/*
 * ca_route_adaptive -- centroid scores and adaptive selection.
 * Paper Section 3.3.2 "Selection", second method: per query cluster a, take
 * key clusters in decreasing estimated attention mass |b| e^{s_ab / sqrt(d)}
 * (the weight the compensation gives a cluster, eq. 21-22; ties to the lower
 * key-cluster index) until their mass reaches `recall` times the total, and
 * at least min(min_count, C) of them (the paper uses 16). Exact greedy
 * selection in fp64 (masses e^{w - w_max}, summed in that order), not the
 * paper's two-pass histogram. Reads centroids->qbar, kbar (16-byte aligned)
 * and count_k. out->k is the capacity of a kept_idx row (k = C_k always
 * suffices; a longer selection is cut at k); out->kept_count is required.
 * recall in [0, 1]; min_count >= 1; C, C_k <= 8192.
 */
ca_status ca_route_adaptive(const ca_shape* shape, const ca_clusters* centroids, double recall,
                            int min_count, const ca_routes* out, void* stream);

/*
 * ca_attend -- block-sparse attention over the kept clusters with striped
 * mean-compensation (SMC) of the excluded ones.
 * Paper Section 1.2 (eq. 5-6) and Appendix A (eq. 21-22): for query i of
 * cluster a,
 *   o_i = ( sum_{b kept} sum_{j in b} e^{q_i.k_j/sqrt(d)} v_j
 *         + sum_{b excluded} |b| e^{q_i.kbar_b/sqrt(d)} vbar_b ) / (same weights)
 * with |b| the member count of key cluster b and vbar_b its mean value.
 * compensate = 0 drops the second sum (plain block-sparse attention).
 * Reads clusters->perm_q/perm_k/count_k/kbar and routes->kept_idx/kept_bits
 * (and routes->kept_count when it is not NULL: per-query-cluster counts, as
 * written by ca_route_adaptive);
 * vbar is computed here. O: device, in shape->layout, written in original
 * row order (padding rows 0). workspace >= ca_attend_workspace_bytes(shape).
 */
ca_status ca_attend(const void* Q, const void* K, const void* V, const ca_shape* shape,
                    const ca_clusters* clusters, const ca_routes* routes, int compensate,
                    void* O, void* workspace, size_t workspace_bytes, void* stream);

/*
 * ca_attend_prepare / ca_attend_prepared -- ca_attend in two halves, for
 * callers that time or schedule the attention kernel on its own.
 * ca_attend_prepare writes into the workspace what the attention reads: the
 * value centroids vbar, the centroid forms the kernels load (bf16 hi/lo
 * parts, fp32 copies, log counts) and, for bf16, the cluster-ordered copies
 * of Q, K and V. ca_attend_prepared then runs the attention (and zeroes O's
 * padding rows) from that workspace; it must follow a ca_attend_prepare on
 * the same stream with the same Q, K, V, clusters and workspace, and reads
 * Q, K, V again only for fp32 inputs. Same arguments, layouts and errors as
 * ca_attend (ca_attend_prepare takes no routes and no O).
 */
ca_status ca_attend_prepare(const void* Q, const void* K, const void* V, const ca_shape* shape,
                            const ca_clusters* clusters, void* workspace, size_t workspace_bytes,
                            void* stream);
ca_status ca_attend_prepared(const void* Q, const void* K, const void* V, const ca_shape* shape,
                             const ca_clusters* clusters, const ca_routes* routes, int compensate,
                             void* O, void* workspace, size_t workspace_bytes, void* stream);

/*
 * ca_dense_attend -- plain softmax(Q K^T / sqrt(d)) V over the n_valid keys
 * (paper eq. 1): the dense baseline the sparse path is measured against.
 * Same layouts as ca_attend. workspace >= ca_dense_workspace_bytes(shape)
 * (may be 0 bytes for shapes that need none).
 */
ca_status ca_dense_attend(const void* Q, const void* K, const void* V, const ca_shape* shape,
                          void* O, void* workspace, size_t workspace_bytes, void* stream);

/*
 * ca_forward -- ca_cluster, ca_route and ca_attend in one call (compensation
 * on when compensate != 0), with every intermediate carved from one
 * workspace of ca_forward_workspace_bytes(shape, k) bytes. `clusters_out` and
 * `routes_out` may be NULL; when given, their buffers receive the
 * intermediates (otherwise they live in the workspace).
 */
ca_status ca_forward(const void* Q, const void* K, const void* V, const ca_shape* shape,
                     const ca_cluster_params* params, int k, int compensate, void* O,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * ca_forward_host -- ca_forward on HOST buffers: copies Q, K, V (host; pinned
 * memory lets the copies overlap the work) into device staging carved from
 * the workspace, runs the forward, copies O back to host, and synchronises
 * before returning. The heads are processed in up to four groups (contiguous
 * ranges of the flattened heads, keyed by their global index as with
 * head_base, so the result equals the whole-layer ca_forward): the copy of a
 * group's inputs overlaps the forward of the previous group, and the copy of
 * a group's output the forward of the next. The forward runs on `stream`;
 * the copies on two short-lived helper streams that start after the work
 * already queued on `stream`. In CA_LAYOUT_BNHD a group of heads is not a
 * contiguous byte range, so the heads form one group (no overlap); the host
 * buffers must hold exactly the call's heads (H_total 0 or H, else
 * CA_ERR_UNSUPPORTED, and the workspace query returns 0).
 * workspace >= ca_forward_host_workspace_bytes(shape, k).
 */
size_t ca_forward_host_workspace_bytes(const ca_shape* shape, int k);
ca_status ca_forward_host(const void* Q_host, const void* K_host, const void* V_host,
                          const ca_shape* shape, const ca_cluster_params* params, int k,
                          int compensate, void* O_host, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * ca_get_device_error -- synchronise `stream` and report (then clear) the
 * device-side error word of the current device: CA_ERR_TIMEOUT if a bounded
 * wait inside a kernel gave up, CA_ERR_CUDA if the stream holds a CUDA error,
 * CA_OK otherwise. The error word is ONE word per device, shared by every
 * stream and every caller of the library in the process: a timeout raised by
 * work on one stream is reported to whichever caller reads the word first
 * (and that read clears it), so callers that share a device and need to
 * attribute errors must serialise their calls and their reads.
 */
ca_status ca_get_device_error(void* stream);

/* Test hook: the time limit, in nanoseconds, of every bounded device-side
 * wait (mbarrier waits on TMA copies and tensor-core work); 0 restores the
 * default of 1 s. Limits above 10 s are rejected with CA_ERR_INVALID_ARG
 * (a longer bound would let a lost arrival hold the GPU). Host only, atomic;
 * affects later launches. */
ca_status ca_set_wait_limit(uint64_t limit_ns);

/* Failure-detection check: launch one CTA on `stream` that waits, through the
 * same bounded mbarrier wait as the attention kernel, on a barrier that
 * completes only when `arrive` is non-zero. With arrive = 0 nothing completes
 * it: the wait gives up after limit_ns nanoseconds and sets CA_ERR_TIMEOUT in
 * the device error word (read it with ca_get_device_error); with arrive != 0
 * the word stays CA_OK. Reads and writes no caller memory. Returns
 * CA_ERR_INVALID_ARG for limit_ns = 0 or above 10 s, CA_ERR_CUDA if the launch
 * fails. */
ca_status ca_check_bounded_wait(uint64_t limit_ns, int arrive, void* stream);

/* Check of the attention kernel's FMA-pipe exponential: writes to y[i] the
 * kernel's own evaluation of 2^x[i] (round-to-nearest split t = n + f, a
 * Remez cubic for 2^f on [-1/2, 1/2], n added to the exponent; inputs below
 * -126 are clamped there). x, y: device fp32 arrays of n elements. Async on
 * `stream`. n = 0 does nothing; CA_ERR_INVALID_ARG for n < 0, or for null
 * pointers with n > 0. */
ca_status ca_check_exp2_poly(const float* x, float* y, int n, void* stream);

/* Number of kernel launches one call makes for this shape (host only):
 * stage 0 = ca_cluster, 1 = ca_route, 2 = ca_attend, 3 = ca_dense_attend;
 * -1 for an invalid shape or stage. */
int ca_launch_count(const ca_shape* shape, int stage);

/* Human-readable name of a status. */
const char* ca_status_string(ca_status status);

/* Library version string. */
const char* ca_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CA_H */
