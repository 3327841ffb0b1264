"""Plain, slow, fp64 CPU oracle of ClusterAttention's forward pass.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product path. It shares
no code with the CUDA library. Both read inputs made by ``workloads``.

Source: "ClusterAttention: A training-free speedup of bidirectional attention"
(arXiv 2608.26965; v1 HTML text and the later revision's text). Citations
below name that paper's sections and equations.

What is computed, per head (Section 3.1 "Overview"; later revision Section 4):
 1. metric matrices M_q = Q^T Q / n (eq. 10-12) and M_k = K_c^T K_c / n with
    column-centred keys (eq. 15 / Appendix B.1);
 2. their PSD square roots by eigendecomposition, small negative eigenvalues
    clamped to 0 (Section 3.2.2 "Key clustering", eq. 13-14);
 3. representations: keys R_q k (eq. 14); queries R_k q / |R_k q| for top-k
    assignment (eq. 16 / eq. 47);
 4. basic recursive splitting (PDDP, Section 3.2.1 "Basic recursive
    splitting"): per set S, sample min(a d, |S|) vectors, power iteration for
    the first principal component warm-started from the parent's estimate and
    a random normal vector, project, put the multiple of c closest to |S|/2
    below the split; repeat until all sets but at most one hold c vectors;
    or diagonalized recursive splitting (Section 3.2.1 "Diagonalized
    recursive splitting"): rotate once into the principal-component basis of
    the full set, then split every set on the coordinate of highest variance
    in its sample;
 5. centroid scores q_bar . k_bar (eq. 18) and top-k selection per query
    cluster (Section 3.3.2 "Selection");
 6. block-sparse attention over the kept clusters with striped
    mean-compensation of every excluded cluster (eq. 21-22, Appendix A);
 7. dense attention softmax(Q K^T / sqrt(d)) V (eq. 1).

Readings where the paper leaves a step open:
 * sample: a systematic sample p_j = floor((j |S| + r) / m), j < m, with the
   offset r drawn by the counter-based generator below; all of S if |S| <= m;
 * power iteration count p = 8 (not stated in the paper);
 * warm start u0 = (u_parent + g_hat) / 2, g_hat = R g / |R g|, g ~ N(0, I)
   drawn in the untransformed coordinates (so the metric can be injected
   without R, Section 6.1 "Improvements"); the root starts from g_hat alone;
 * ties: equal projections are ordered by original token index, the lower
   side of every split is the left child; the split count rule picks the
   smaller multiple of c on an exact tie;
 * selection: exact top-k (ties to the lower key-cluster index), not the
   paper's approximate histogram; adaptive selection as the exact greedy
   prefix by estimated mass |b| e^{s_ab / sqrt(d)} (see adaptive_route);
 * compensation weight |c| is the number of real members of the cluster;
 * diagonalized splitting: the basis diagonalises the (centred) covariance
   of the representations over all valid rows; basis vectors are ordered by
   descending eigenvalue and signed so that the raw-space direction R u_j
   has its largest-magnitude entry positive (a sign that does not depend on
   which root of the metric forms the representation); the per-set sample is
   the basic splitting's, and the highest sample variance picks the
   coordinate (lowest index on a tie).

Random numbers: SplitMix64 (Steele, Lea & Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014) on a per-node counter, turned
into normals by the Box-Muller transform. The CUDA side implements the same
published generator independently.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np

__all__ = [
    "splitmix64", "node_key", "sample_offset", "node_gaussian",
    "metric_matrices", "psd_root", "key_representation", "query_representation",
    "split_count", "plan_tree", "num_clusters",
    "PddpResult", "pddp_partition", "pddp_partition_metric_form",
    "pca_basis", "diagonal_partition",
    "HeadClusters", "cluster_head", "cluster_workload",
    "centroid_scores", "topk_route", "route_bits",
    "compensated_attention", "dense_attention",
    "ForwardResult", "forward_head",
]

MASK64 = (1 << 64) - 1
SAMPLE_TAG = 0x5A3C_96E1_0F87_D2B4   # separates the sample-offset draw from the normals


# ---------------------------------------------------------------------------
# Counter-based generator (SplitMix64 finaliser + Box-Muller).
# ---------------------------------------------------------------------------

def splitmix64(x: int) -> int:
    """One SplitMix64 step: add the golden-gamma increment, then mix."""
    z = (x + 0x9E3779B97F4A7C15) & MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def node_key(seed: int, bh: int, tensor: int, heap: int) -> int:
    """Stream key of one recursion node.

    bh = b * H + h; tensor 0 = queries, 1 = keys; heap = heap index of the
    node (root 1, children 2i and 2i+1).
    """
    x = splitmix64(seed & MASK64)
    x = splitmix64(x ^ (bh & MASK64))
    return splitmix64(x ^ (((tensor & 0xFFFF) << 48) | (heap & ((1 << 48) - 1))))


def sample_offset(key: int, size: int) -> int:
    """Offset r in [0, size) of the node's systematic sample."""
    return splitmix64(key ^ SAMPLE_TAG) % size


def node_gaussian(key: int, d: int) -> np.ndarray:
    """d standard normal draws of one node (Box-Muller, cosine branch)."""
    g = np.empty(d)
    for j in range(d):
        a = splitmix64((key + 2 * j + 1) & MASK64)
        b = splitmix64((key + 2 * j + 2) & MASK64)
        u1 = ((a >> 11) + 1) * 2.0 ** -53      # (0, 1]
        u2 = (b >> 11) * 2.0 ** -53            # [0, 1)
        g[j] = math.sqrt(-2.0 * math.log(u1)) * math.cos(2.0 * math.pi * u2)
    return g


# ---------------------------------------------------------------------------
# S1 / transforms: metric matrices and their roots.
# ---------------------------------------------------------------------------

def metric_matrices(Q: np.ndarray, K: np.ndarray):
    """Metric matrices of one head (valid rows only, fp64).

    M_q = Q^T Q / n: average squared logit difference of two keys over the
    queries (Section 3.2.2, eq. 10-12).
    M_k = K_c^T K_c / n with K_c the column-centred keys (eq. 15, Appendix B.1
    eq. 37, Appendix B.2 eq. 46).
    Returns (M_q, M_k, k_mean).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    n = Q.shape[0]
    M_q = Q.T @ Q / n
    k_mean = K.mean(axis=0)
    Kc = K - k_mean
    M_k = Kc.T @ Kc / n
    return M_q, M_k, k_mean


def psd_root(M: np.ndarray) -> np.ndarray:
    """Symmetric root R with R R = M, from an eigendecomposition; negative
    eigenvalues (numerical noise) are clamped to 0 (Section 3.2.2)."""
    lam, U = np.linalg.eigh(M)
    lam = np.maximum(lam, 0.0)
    return (U * np.sqrt(lam)) @ U.T


def key_representation(K: np.ndarray, R_q: np.ndarray) -> np.ndarray:
    """Keys mapped to query space: y = R_q k (eq. 14)."""
    return np.asarray(K, dtype=np.float64) @ R_q.T


def query_representation_adaptive(Q: np.ndarray, R_k: np.ndarray) -> np.ndarray:
    """Query representation for adaptive selection: R_k q (eq. 15), under
    which |R_k (q1 - q2)|^2 = (q1 - q2)^T K_c^T K_c (q1 - q2) / n; no
    normalisation (Section 3.2.2 "Query clustering", first case)."""
    return np.asarray(Q, dtype=np.float64) @ R_k.T


def query_representation(Q: np.ndarray, R_k: np.ndarray) -> np.ndarray:
    """Top-k query representation r(q) = R_k q / |R_k q| (eq. 16, eq. 47).
    A query with R_k q = 0 maps to the zero vector."""
    Y = np.asarray(Q, dtype=np.float64) @ R_k.T
    nrm = np.sqrt(np.einsum("ij,ij->i", Y, Y))
    out = np.zeros_like(Y)
    nz = nrm > 0
    out[nz] = Y[nz] / nrm[nz, None]
    return out


# ---------------------------------------------------------------------------
# Tree shape: the multiple of c closest to |S|/2 goes below the split.
# ---------------------------------------------------------------------------

def split_count(size: int, c: int) -> int:
    """Number of vectors put below the split of a set of ``size`` vectors:
    the multiple of c closest to size/2 (Section 3.2.1), the smaller one on
    an exact tie."""
    j_lo = size // (2 * c)
    j_hi = -(-size // (2 * c))
    t_lo, t_hi = c * j_lo, c * j_hi
    if abs(2 * t_hi - size) < abs(2 * t_lo - size):
        return t_hi
    return t_lo


def num_clusters(n: int, c: int) -> int:
    return -(-n // c)


def plan_tree(n: int, c: int):
    """All nodes of the recursion, depth first, left child first.

    Each node is (heap, depth, offset, size, t); t = 0 for leaves.
    ``offset`` is the node's first slot in the final left-to-right leaf order.
    """
    nodes = []

    def rec(heap, depth, off, size):
        if size <= c:
            nodes.append((heap, depth, off, size, 0))
            return
        t = split_count(size, c)
        nodes.append((heap, depth, off, size, t))
        rec(2 * heap, depth + 1, off, t)
        rec(2 * heap + 1, depth + 1, off + t, size - t)

    rec(1, 0, 0, n)
    return nodes


# ---------------------------------------------------------------------------
# Basic recursive splitting (PDDP).
# ---------------------------------------------------------------------------

@dataclass
class PddpResult:
    leaves: List[np.ndarray]                 # member original indices, ascending, left to right
    min_margin: float = math.inf             # smallest relative gap at a split
    splits: list = field(default_factory=list)  # (heap, size, t, lower_max, upper_min, u)


def _sample_positions(size: int, m: int, key: int) -> np.ndarray:
    if size <= m:
        return np.arange(size)
    r = sample_offset(key, size)
    j = np.arange(m, dtype=np.int64)
    return (j * size + r) // m


def pddp_partition(Y: np.ndarray, R: np.ndarray, c: int, *, seed: int, bh: int,
                   tensor: int, power_iters: int = 8, sample_factor: int = 1,
                   record: bool = False) -> PddpResult:
    """Basic recursive splitting of the rows of Y (already transformed).

    Y: [n, d] representations in original token order. R: the root used to
    transform the random warm-start vector (identity for no transform).
    Follows Section 3.2.1: sample min(a d, |S|) vectors, estimate the first
    principal component of the sample by power iteration warm-started from the
    mean of the parent's estimate and a random normal vector of the parent's
    (unit) norm, project all of S, split with the multiple of c closest to
    |S|/2 below; recurse until sets hold at most c vectors.
    """
    Y = np.asarray(Y, dtype=np.float64)
    n, d = Y.shape
    res = PddpResult(leaves=[])
    m_cap = sample_factor * d

    def rec(members: np.ndarray, heap: int, u_parent: Optional[np.ndarray]):
        size = members.shape[0]
        if size <= c:
            res.leaves.append(members)
            return
        key = node_key(seed, bh, tensor, heap)
        m = min(m_cap, size)
        pos = _sample_positions(size, m, key)
        Ys = Y[members[pos]]
        Yc = Ys - Ys.mean(axis=0)
        Cy = Yc.T @ Yc / m                       # sample covariance
        Rg = R @ node_gaussian(key, d)
        gn = math.sqrt(float(Rg @ Rg))
        g_hat = Rg / gn if gn > 0 else np.zeros(d)
        u = g_hat if u_parent is None else 0.5 * (u_parent + g_hat)
        for _ in range(power_iters):             # power iteration
            v = Cy @ u
            vn = math.sqrt(float(v @ v))
            u = v / vn if vn > 0 else np.zeros(d)
        proj = Y[members] @ u + 0.0              # + 0.0 turns -0.0 into +0.0
        t = split_count(size, c)
        order = np.lexsort((members, proj))      # by projection, then by index
        lo_sorted = proj[order]
        spread = float(lo_sorted[-1] - lo_sorted[0])
        gap = float(lo_sorted[t] - lo_sorted[t - 1])
        margin = gap / spread if spread > 0 else 0.0
        res.min_margin = min(res.min_margin, margin)
        if record:
            res.splits.append((heap, size, t, float(lo_sorted[t - 1]),
                               float(lo_sorted[t]), u.copy()))
        lower = np.sort(members[order[:t]])
        upper = np.sort(members[order[t:]])
        rec(lower, 2 * heap, u)
        rec(upper, 2 * heap + 1, u)

    rec(np.arange(n), 1, None)
    return res


def pddp_partition_metric_form(X: np.ndarray, M: np.ndarray, c: int, *, seed: int,
                               bh: int, tensor: int, power_iters: int = 8,
                               sample_factor: int = 1) -> PddpResult:
    """The same recursion with the metric injected into the power iteration
    instead of transforming the vectors (Section 6.1 "Improvements": no
    eigendecomposition). X holds untransformed vectors (queries already divided
    by |R_k q|); u = R z is never formed: C_y u = R C_x M z, |u|^2 = z^T M z,
    and the projection y . u = x^T M z. Used only to check that the literal
    form and the injected form give one partition.
    """
    X = np.asarray(X, dtype=np.float64)
    n, d = X.shape
    res = PddpResult(leaves=[])
    m_cap = sample_factor * d

    def rec(members, heap, z_parent):
        size = members.shape[0]
        if size <= c:
            res.leaves.append(members)
            return
        key = node_key(seed, bh, tensor, heap)
        m = min(m_cap, size)
        pos = _sample_positions(size, m, key)
        Xs = X[members[pos]]
        Xc = Xs - Xs.mean(axis=0)
        g = node_gaussian(key, d)
        gq = float(g @ M @ g)
        g_hat = g / math.sqrt(gq) if gq > 0 else np.zeros(d)
        z = g_hat if z_parent is None else 0.5 * (z_parent + g_hat)
        for _ in range(power_iters):
            z = Xc.T @ (Xc @ (M @ z)) / m
            q = float(z @ M @ z)
            z = z / math.sqrt(q) if q > 0 else np.zeros(d)
        proj = X[members] @ (M @ z) + 0.0
        t = split_count(size, c)
        order = np.lexsort((members, proj))
        lower = np.sort(members[order[:t]])
        upper = np.sort(members[order[t:]])
        rec(lower, 2 * heap, z)
        rec(upper, 2 * heap + 1, z)

    rec(np.arange(n), 1, None)
    return res


# ---------------------------------------------------------------------------
# Diagonalized recursive splitting.
# ---------------------------------------------------------------------------

def pca_basis(Y: np.ndarray, factor: Optional[np.ndarray] = None) -> tuple:
    """Principal-component basis of the representations Y (rows, the full
    set) from the eigendecomposition of their covariance (Section 3.2.1
    "Diagonalized recursive splitting"; later revision Section 4.1.1).

    Y holds the rows x F of the raw rows x (F = ``factor``, the identity when
    None). Returns (U, lam): the columns of U are unit eigenvectors ordered by
    descending eigenvalue lam (ties keep the solver's order), each signed so
    that the raw-space direction w_j = F u_j (coordinate j of a row is
    x . w_j) has its entry of largest magnitude (the first on an exact tie)
    positive; this fixes which side of a split is "below", and w_j is the
    same for every factor F with F F^T equal to the metric.
    """
    Y = np.asarray(Y, dtype=np.float64)
    n = Y.shape[0]
    Yc = Y - Y.mean(axis=0)
    cov = Yc.T @ Yc / n
    lam, U = np.linalg.eigh(cov)
    order = np.argsort(-lam, kind="stable")
    lam, U = lam[order], U[:, order].copy()
    Wd = U if factor is None else np.asarray(factor, dtype=np.float64) @ U
    for j in range(U.shape[1]):
        i = int(np.argmax(np.abs(Wd[:, j])))
        if Wd[i, j] < 0:
            U[:, j] = -U[:, j]
    return U, lam


def diagonal_partition(Y: np.ndarray, c: int, *, seed: int, bh: int, tensor: int,
                       sample_factor: int = 1, record: bool = False,
                       factor: Optional[np.ndarray] = None) -> PddpResult:
    """Diagonalized recursive splitting of the rows of Y (already transformed,
    Y = X F with ``factor`` F; the identity when None).

    The rows are rotated once into the principal-component basis of the full
    set, Z = Y U (pca_basis). At every set S: take the same sample of
    min(a d, |S|) members as the basic splitting (a = sample_factor), find
    the coordinate whose variance over the sample is highest (the lowest
    coordinate index on an exact tie) and split S on that coordinate with the
    multiple of c closest to |S|/2 below, equal values ordered by token
    index; recurse until sets hold at most c vectors.
    """
    Y = np.asarray(Y, dtype=np.float64)
    n, d = Y.shape
    U, _ = pca_basis(Y, factor)
    Z = Y @ U
    res = PddpResult(leaves=[])
    m_cap = sample_factor * d

    def rec(members: np.ndarray, heap: int):
        size = members.shape[0]
        if size <= c:
            res.leaves.append(members)
            return
        key = node_key(seed, bh, tensor, heap)
        m = min(m_cap, size)
        Zs = Z[members[_sample_positions(size, m, key)]]
        var = ((Zs - Zs.mean(axis=0)) ** 2).mean(axis=0)
        j = int(np.argmax(var))                   # first maximum on ties
        proj = Z[members, j] + 0.0
        t = split_count(size, c)
        order = np.lexsort((members, proj))
        srt = proj[order]
        spread = float(srt[-1] - srt[0])
        margin = float(srt[t] - srt[t - 1]) / spread if spread > 0 else 0.0
        res.min_margin = min(res.min_margin, margin)
        if record:
            res.splits.append((heap, size, t, float(srt[t - 1]), float(srt[t]), j))
        rec(np.sort(members[order[:t]]), 2 * heap)
        rec(np.sort(members[order[t:]]), 2 * heap + 1)

    rec(np.arange(n), 1)
    return res


# ---------------------------------------------------------------------------
# Clustering of one head: transforms + PDDP + centroids.
# ---------------------------------------------------------------------------

@dataclass
class HeadClusters:
    perm_q: np.ndarray      # [C*c] int32, original token per slot, -1 in pad slots
    perm_k: np.ndarray
    count_q: np.ndarray     # [C] int32
    count_k: np.ndarray
    qbar: np.ndarray        # [C, d] fp64 centroids in original space
    kbar: np.ndarray
    min_margin_q: float
    min_margin_k: float


def _leaves_to_perm(leaves: Sequence[np.ndarray], c: int):
    C = len(leaves)
    perm = np.full(C * c, -1, dtype=np.int32)
    counts = np.zeros(C, dtype=np.int32)
    for a, mem in enumerate(leaves):
        perm[a * c: a * c + mem.shape[0]] = mem
        counts[a] = mem.shape[0]
    return perm, counts


def _centroids(X: np.ndarray, leaves: Sequence[np.ndarray]) -> np.ndarray:
    """Cluster means in the original (untransformed) space (eq. 18)."""
    X = np.asarray(X, dtype=np.float64)
    return np.stack([X[mem].mean(axis=0) for mem in leaves])


def cluster_head(Q: np.ndarray, K: np.ndarray, c: int, *, seed: int = 0, bh: int = 0,
                 power_iters: int = 8, sample_factor: int = 1,
                 transform: bool = True, query_form: str = "topk",
                 splitting: str = "basic", c_k: Optional[int] = None) -> HeadClusters:
    """Cluster the valid queries and keys of one head (rows [n, d]).

    Keys are split in the query-aware space R_q k; queries in the key-aware,
    normalised space R_k q / |R_k q| (top-k form, eq. 16) or, with
    ``query_form="adaptive"``, in R_k q (eq. 15). ``transform=False`` splits
    the raw vectors (R = I, no normalisation), the paper's ablation.
    ``splitting`` is "basic" (power iteration per set) or "diagonal"
    (one principal-component rotation, coordinate splits). ``c`` is the
    query cluster size; ``c_k`` the key cluster size (``c`` when None), the
    paper evaluating 64 for queries and 128 for keys (Section 3.1): each
    tensor's tree follows its own size.
    """
    ck = c if c_k is None else c_k
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    d = Q.shape[1]
    if transform:
        M_q, M_k, _ = metric_matrices(Q, K)
        R_q = psd_root(M_q)
        R_k = psd_root(M_k)
        Yk = key_representation(K, R_q)
        Yq = (query_representation(Q, R_k) if query_form == "topk"
              else query_representation_adaptive(Q, R_k))
    else:
        R_q = R_k = np.eye(d)
        Yk, Yq = K, Q
    if splitting == "diagonal":
        # Y = X R with R symmetric (query rows also scaled by 1 / |R_k q|)
        rq = diagonal_partition(Yq, c, seed=seed, bh=bh, tensor=0, sample_factor=sample_factor, factor=R_k)
        rk = diagonal_partition(Yk, ck, seed=seed, bh=bh, tensor=1, sample_factor=sample_factor, factor=R_q)
    else:
        rq = pddp_partition(Yq, R_k, c, seed=seed, bh=bh, tensor=0,
                            power_iters=power_iters, sample_factor=sample_factor)
        rk = pddp_partition(Yk, R_q, ck, seed=seed, bh=bh, tensor=1,
                            power_iters=power_iters, sample_factor=sample_factor)
    perm_q, count_q = _leaves_to_perm(rq.leaves, c)
    perm_k, count_k = _leaves_to_perm(rk.leaves, ck)
    return HeadClusters(perm_q=perm_q, perm_k=perm_k, count_q=count_q, count_k=count_k,
                        qbar=_centroids(Q, rq.leaves), kbar=_centroids(K, rk.leaves),
                        min_margin_q=rq.min_margin, min_margin_k=rk.min_margin)


def random_leaves(n: int, c: int, *, seed: int, bh: int, tensor: int) -> List[np.ndarray]:
    """Random clusters, the baseline of the paper's error analysis (Section
    4, "random clustering and top-k" against the recursive split): token i
    draws the counter-based key splitmix64(node_key(seed, bh, tensor, 0) ^ i)
    (heap index 0 belongs to no node of the split tree); the tokens ordered
    by (key, index) are cut into consecutive groups of c, the remainder group
    last, members ascending."""
    base = node_key(seed, bh, tensor, 0)
    keys = np.array([splitmix64(base ^ i) for i in range(n)], dtype=np.uint64)
    order = np.lexsort((np.arange(n), keys))
    return [np.sort(order[a:a + c]) for a in range(0, n, c)]


def cluster_head_random(Q: np.ndarray, K: np.ndarray, c: int, *, seed: int = 0, bh: int = 0,
                        c_k: Optional[int] = None) -> HeadClusters:
    """Random clusters of the valid queries and keys of one head, with the
    same outputs as cluster_head (permutation, counts, centroids); keys in
    groups of ``c_k`` (``c`` when None)."""
    ck = c if c_k is None else c_k
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    n = Q.shape[0]
    lq = random_leaves(n, c, seed=seed, bh=bh, tensor=0)
    lk = random_leaves(n, ck, seed=seed, bh=bh, tensor=1)
    perm_q, count_q = _leaves_to_perm(lq, c)
    perm_k, count_k = _leaves_to_perm(lk, ck)
    return HeadClusters(perm_q=perm_q, perm_k=perm_k, count_q=count_q, count_k=count_k,
                        qbar=_centroids(Q, lq), kbar=_centroids(K, lk),
                        min_margin_q=float("inf"), min_margin_k=float("inf"))


def cluster_workload(Q: np.ndarray, K: np.ndarray, n_valid: int, c: int, *, seed: int = 0,
                     power_iters: int = 8, heads: Optional[Sequence[int]] = None,
                     transform: bool = True, splitting: str = "basic",
                     query_form: str = "topk", c_k: Optional[int] = None) -> List[HeadClusters]:
    """Cluster every (b, h) of [B, H, N_alloc, d] inputs; rows >= n_valid are padding."""
    B, H = Q.shape[:2]
    out = []
    for b in range(B):
        for h in range(H):
            bh = b * H + h
            if heads is not None and bh not in heads:
                continue
            out.append(cluster_head(Q[b, h, :n_valid], K[b, h, :n_valid], c, seed=seed,
                                    bh=bh, power_iters=power_iters, transform=transform,
                                    splitting=splitting, query_form=query_form, c_k=c_k))
    return out


# ---------------------------------------------------------------------------
# Assignment: centroid scores and top-k.
# ---------------------------------------------------------------------------

def centroid_scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """s_ab = q_bar_a . k_bar_b, the mean pairwise logit (eq. 18), fp64."""
    return np.asarray(qbar, np.float64) @ np.asarray(kbar, np.float64).T


def topk_route(scores: np.ndarray, k: int) -> np.ndarray:
    """Per query cluster, the k key clusters with the largest score (ties to
    the lower key-cluster index), listed in ascending order (Section 3.3.2)."""
    Cq, Ck = scores.shape
    idx = np.arange(Ck)
    kept = np.empty((Cq, k), dtype=np.int32)
    for a in range(Cq):
        order = np.lexsort((idx, -scores[a]))
        kept[a] = np.sort(order[:k])
    return kept


def cluster_log_mass(scores: np.ndarray, count_k: np.ndarray, d: int) -> np.ndarray:
    """Log of the estimated attention mass of key cluster b for query cluster
    a: |b| e^{s_ab / sqrt(d)}, the weight the compensation gives an excluded
    cluster (eq. 21-22), with s_ab the centroid score (eq. 18)."""
    return (np.asarray(scores, np.float64) * (1.0 / math.sqrt(d))
            + np.log(np.asarray(count_k, np.float64))[None, :])


def adaptive_route(scores: np.ndarray, count_k: np.ndarray, d: int, recall: float,
                   min_count: int = 16) -> List[np.ndarray]:
    """Adaptive selection (Section 3.3.2 "Selection"): per query cluster, take
    key clusters in decreasing estimated attention mass (ties to the lower
    key-cluster index) until their mass reaches ``recall`` times the total,
    and at least ``min_count`` of them (16 in the paper). Exact greedy
    reading of the paper's histogram approximation: masses are
    e^{w_b - max w} in fp64 with w = cluster_log_mass, summed in that order.
    Returns one ascending int32 array per query cluster."""
    W = cluster_log_mass(scores, count_k, d)
    Cq, Ck = W.shape
    idx = np.arange(Ck)
    out = []
    for a in range(Cq):
        order = np.lexsort((idx, -W[a]))
        mass = np.exp(W[a, order] - W[a, order[0]])
        cum = np.cumsum(mass)
        hit = cum >= recall * cum[-1]
        k = (int(np.argmax(hit)) + 1 if hit.any() else Ck) if recall > 0 else 1
        k = max(k, min(min_count, Ck))
        out.append(np.sort(order[:k]).astype(np.int32))
    return out


def route_bits(kept: np.ndarray, Ck: int) -> np.ndarray:
    """Kept list as a bitmask [Cq, ceil(Ck/32)] uint32 (bit b%32 of word b//32)."""
    Cq = len(kept)
    W = -(-Ck // 32)
    bits = np.zeros((Cq, W), dtype=np.uint64)
    for a in range(Cq):
        for b in kept[a]:
            bits[a, b // 32] |= np.uint64(1) << np.uint64(b % 32)
    return bits.astype(np.uint32)


# ---------------------------------------------------------------------------
# Attention.
# ---------------------------------------------------------------------------

def _members(perm: np.ndarray, count: np.ndarray, c: int, a: int) -> np.ndarray:
    return perm[a * c: a * c + count[a]].astype(np.int64)


def compensated_attention(Q, K, V, perm_q, count_q, perm_k, count_k, kept, c: int, *,
                          compensate: bool = True, clusters: Optional[Sequence[int]] = None,
                          n_out: Optional[int] = None, c_k: Optional[int] = None) -> np.ndarray:
    """Block-sparse attention over the kept key clusters, with striped
    mean-compensation of every excluded key cluster (eq. 21-22).

    For query i of cluster a:
      o_i = (sum_{b kept} sum_{j in b} e^{l_ij} v_j
             + sum_{b excluded} |b| e^{q_i . k_bar_b / sqrt(d)} v_bar_b) / (same weights)
    with l_ij = q_i . k_j / sqrt(d); ``compensate=False`` drops the second sum.
    ``c`` is the slot size of perm_q, ``c_k`` that of perm_k (``c`` when None).
    Returns O [n_out, d] in original token order (rows of clusters not
    evaluated are left at 0).
    """
    Q = np.asarray(Q, np.float64); K = np.asarray(K, np.float64); V = np.asarray(V, np.float64)
    d = Q.shape[1]
    scale = 1.0 / math.sqrt(d)
    Cq = count_q.shape[0]
    Ck = count_k.shape[0]
    kmem = [_members(perm_k, count_k, c if c_k is None else c_k, b) for b in range(Ck)]
    kbar = np.stack([K[m].mean(axis=0) for m in kmem])
    vbar = np.stack([V[m].mean(axis=0) for m in kmem])
    logcnt = np.log(count_k.astype(np.float64))
    O = np.zeros((n_out if n_out is not None else Q.shape[0], d))
    for a in (range(Cq) if clusters is None else clusters):
        qm = _members(perm_q, count_q, c, a)
        qa = Q[qm]
        kept_a = np.asarray(kept[a], dtype=np.int64)
        J = np.concatenate([kmem[b] for b in kept_a])
        logits = (qa @ K[J].T) * scale
        vals = V[J]
        if compensate:
            excl = np.setdiff1d(np.arange(Ck), kept_a)
            if excl.size:
                lc = (qa @ kbar[excl].T) * scale + logcnt[excl]
                logits = np.concatenate([logits, lc], axis=1)
                vals = np.concatenate([vals, vbar[excl]], axis=0)
        mx = logits.max(axis=1, keepdims=True)
        w = np.exp(logits - mx)
        O[qm] = (w @ vals) / w.sum(axis=1, keepdims=True)
    return O


def dense_attention(Q, K, V, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """softmax(Q K^T / sqrt(d)) V over all valid keys (eq. 1), fp64."""
    Q = np.asarray(Q, np.float64); K = np.asarray(K, np.float64); V = np.asarray(V, np.float64)
    d = Q.shape[1]
    q = Q if rows is None else Q[rows]
    out = np.empty((q.shape[0], d))
    step = 256
    for s in range(0, q.shape[0], step):
        lg = (q[s:s + step] @ K.T) / math.sqrt(d)
        lg -= lg.max(axis=1, keepdims=True)
        w = np.exp(lg)
        out[s:s + step] = (w @ V) / w.sum(axis=1, keepdims=True)
    return out


# ---------------------------------------------------------------------------
# Whole forward of one head.
# ---------------------------------------------------------------------------

@dataclass
class ForwardResult:
    clusters: HeadClusters
    kept: np.ndarray
    O: np.ndarray


def forward_head(Q, K, V, c: int, k: int, *, seed: int = 0, bh: int = 0,
                 power_iters: int = 8, compensate: bool = True,
                 clusters_subset: Optional[Sequence[int]] = None,
                 transform: bool = True, c_k: Optional[int] = None) -> ForwardResult:
    """cluster -> route -> attend for one head's valid rows [n, d]; ``c`` is
    the query cluster size, ``c_k`` the key cluster size (``c`` when None)."""
    hc = cluster_head(Q, K, c, seed=seed, bh=bh, power_iters=power_iters, transform=transform, c_k=c_k)
    kept = topk_route(centroid_scores(hc.qbar, hc.kbar), k)
    O = compensated_attention(Q, K, V, hc.perm_q, hc.count_q, hc.perm_k, hc.count_k, kept, c,
                              compensate=compensate, clusters=clusters_subset, c_k=c_k)
    return ForwardResult(clusters=hc, kept=kept, O=O)
