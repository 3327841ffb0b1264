"""Pins of the fp64 oracle against what the paper and the mathematics fix.

Each test checks the oracle against something other than itself: an identity
derived in the paper, a brute-force evaluation of a definition on tiny inputs,
a textbook special case, or a library routine. Paper citations name sections
and equations of "ClusterAttention: A training-free speedup of bidirectional
attention".
"""
import math
import os

import numpy as np
import pytest

from oracle import ca_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# Counter-based generator
# ---------------------------------------------------------------------------

def test_splitmix64_published_sequence():
    # First three outputs of SplitMix64 seeded with state 0 (the generator's
    # published reference sequence): state advances by the golden gamma.
    gamma = 0x9E3779B97F4A7C15
    assert orc.splitmix64(0) == 0xE220A8397B1DCDAF
    assert orc.splitmix64(gamma) == 0x6E789E6AA1B965F4
    assert orc.splitmix64((2 * gamma) & orc.MASK64) == 0x06C45D188009454F


def test_node_gaussian_is_standard_normal():
    draws = np.concatenate([orc.node_gaussian(orc.node_key(7, bh, 0, heap), 64)
                            for bh in range(4) for heap in range(1, 65)])
    assert draws.shape == (16384,)
    assert abs(draws.mean()) < 0.05
    assert abs(draws.var() - 1.0) < 0.05
    # Distinct nodes draw distinct vectors.
    a = orc.node_gaussian(orc.node_key(7, 0, 0, 2), 8)
    b = orc.node_gaussian(orc.node_key(7, 0, 0, 3), 8)
    assert not np.allclose(a, b)


# ---------------------------------------------------------------------------
# Metrics and transforms (Section 3.2.2, Appendix B)
# ---------------------------------------------------------------------------

def test_key_metric_is_average_squared_logit_difference_eq10():
    # eq. 10-11: d_q(k1,k2)^2 = |Q(k1-k2)|^2/n, evaluated here query by query.
    r = rng(1)
    Q = r.standard_normal((37, 6)); K = r.standard_normal((11, 6))
    M_q, _, _ = orc.metric_matrices(Q, K)
    R_q = orc.psd_root(M_q)
    Y = orc.key_representation(K, R_q)
    for i in range(K.shape[0]):
        for j in range(K.shape[0]):
            brute = sum((float(q @ K[i]) - float(q @ K[j])) ** 2 for q in Q) / Q.shape[0]
            assert abs(float(np.sum((Y[i] - Y[j]) ** 2)) - brute) < 1e-12 * max(1.0, brute)


def test_root_squares_to_metric_and_clamps_negative_eigenvalues():
    r = rng(2)
    A = r.standard_normal((50, 8))
    M = A.T @ A / 50
    R = orc.psd_root(M)
    assert np.allclose(R, R.T, atol=1e-14)
    assert np.allclose(R @ R, M, rtol=0, atol=1e-12)
    # A symmetric matrix with a negative eigenvalue: the root squares to the
    # matrix with that eigenvalue set to 0.
    U, _ = np.linalg.qr(r.standard_normal((5, 5)))
    lam = np.array([3.0, 1.0, 0.5, 0.0, -0.25])
    Mneg = (U * lam) @ U.T
    Rn = orc.psd_root(Mneg)
    assert np.allclose(Rn @ Rn, (U * np.maximum(lam, 0)) @ U.T, rtol=0, atol=1e-12)


def test_centred_key_metric_equals_pair_difference_gram_eq46():
    # Appendix B.2, eq. 42-46: D^T D over all ordered key pairs = 2 n K_c^T K_c.
    r = rng(3)
    K = r.standard_normal((9, 4)) + 3.0
    Q = r.standard_normal((9, 4))
    n = K.shape[0]
    _, M_k, kmean = orc.metric_matrices(Q, K)
    D = np.array([K[a] - K[b] for a in range(n) for b in range(n)])
    assert np.allclose(D.T @ D, 2 * n * (n * M_k), rtol=1e-12, atol=1e-10)
    assert np.allclose(kmean, [K[:, j].sum() / n for j in range(4)], atol=1e-14)


def test_query_representation_unit_norm_and_scale_invariant():
    r = rng(4)
    Q = r.standard_normal((64, 8)); K = r.standard_normal((64, 8))
    _, M_k, _ = orc.metric_matrices(Q, K)
    R_k = orc.psd_root(M_k)
    Y = orc.query_representation(Q, R_k)
    assert np.allclose(np.linalg.norm(Y, axis=1), 1.0, atol=1e-14)
    alpha = r.uniform(0.1, 10.0, size=(64, 1))
    Y2 = orc.query_representation(alpha * Q, R_k)
    assert np.allclose(Y, Y2, atol=1e-13)


def test_query_scaling_leaves_clustering_unchanged():
    # eq. 16: only the direction of R_k q matters, so rescaling queries by
    # positive factors changes neither the partition nor the key clustering
    # (M_q changes, so keys are compared in a rescaled metric: key clusters
    # may change; the query clusters may not).
    r = rng(5)
    Q = r.standard_normal((512, 8)); K = r.standard_normal((512, 8))
    hc1 = orc.cluster_head(Q, K, 64, seed=3)
    alpha = np.exp(r.uniform(-1, 1, size=(512, 1)))
    hc2 = orc.cluster_head(alpha * Q, K, 64, seed=3)
    assert np.array_equal(hc1.perm_q, hc2.perm_q)


def test_query_shift_in_key_null_direction_leaves_clustering_unchanged_eq38():
    # eq. 36-38: a shift delta with K_c delta = 0 changes no attention weight and
    # no query representation. Keys constant along axis 0 make K_c e_0 = 0.
    r = rng(6)
    n, d = 512, 8
    K = r.standard_normal((n, d)); K[:, 0] = 1.5
    Q = r.standard_normal((n, d))
    _, M_k, _ = orc.metric_matrices(Q, K)
    R_k = orc.psd_root(M_k)
    delta = np.zeros(d); delta[0] = 1.0
    shifts = r.uniform(-3, 3, size=(n, 1)) * delta
    assert np.allclose(orc.query_representation(Q, R_k),
                       orc.query_representation(Q + shifts, R_k), atol=1e-6)
    hc1 = orc.cluster_head(Q, K, 64, seed=1)
    hc2 = orc.cluster_head(Q + shifts, K, 64, seed=1)
    assert np.array_equal(hc1.perm_q, hc2.perm_q)


# ---------------------------------------------------------------------------
# Tree shape (Section 3.1, 3.2.1)
# ---------------------------------------------------------------------------

def _golden_shapes():
    rows = []
    with open(os.path.join(GOLDEN, "tree_shapes.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(tuple(int(x) for x in line.split()))
    return rows


@pytest.mark.parametrize("n,c,C,last,root_t", _golden_shapes())
def test_tree_shape_golden(n, c, C, last, root_t):
    assert orc.split_count(n, c) == root_t
    nodes = orc.plan_tree(n, c)
    leaves = [nd for nd in nodes if nd[4] == 0]
    assert len(leaves) == C == orc.num_clusters(n, c)
    sizes = [nd[3] for nd in sorted(leaves, key=lambda x: x[2])]
    assert sizes[:-1] == [c] * (C - 1)
    assert sizes[-1] == last
    # Every split puts a multiple of c below it.
    for heap, depth, off, size, t in nodes:
        if t:
            assert t % c == 0 and 0 < t < size


# ---------------------------------------------------------------------------
# PDDP (Section 3.2.1)
# ---------------------------------------------------------------------------

def _mixture(r, n, d, comps=8, std=0.3):
    mu = r.standard_normal((comps, d))
    z = r.integers(0, comps, n)
    return mu[z] + std * r.standard_normal((n, d))


@pytest.mark.parametrize("n,c", [(1024, 64), (1000, 64), (777, 128), (300, 64), (128, 64)])
def test_pddp_partition_is_bijection_with_fixed_sizes(n, c):
    r = rng(7)
    Q = _mixture(r, n, 16); K = _mixture(r, n, 16)
    hc = orc.cluster_head(Q, K, c, seed=11)
    C = orc.num_clusters(n, c)
    for perm, cnt in ((hc.perm_q, hc.count_q), (hc.perm_k, hc.count_k)):
        assert perm.shape == (C * c,)
        real = perm[perm >= 0]
        assert np.array_equal(np.sort(real), np.arange(n))
        assert list(cnt[:-1]) == [c] * (C - 1) and cnt[-1] == n - (C - 1) * c
        for a in range(C):
            seg = perm[a * c:(a + 1) * c]
            assert np.all(seg[:cnt[a]] >= 0) and np.all(seg[cnt[a]:] == -1)
            assert np.all(np.diff(seg[:cnt[a]]) > 0)   # ascending original index


def test_pddp_every_split_orders_projections():
    r = rng(8)
    Y = _mixture(r, 1000, 8)
    res = orc.pddp_partition(Y, np.eye(8), 64, seed=2, bh=0, tensor=1, record=True)
    assert len(res.splits) == orc.num_clusters(1000, 64) - 1
    for heap, size, t, lower_max, upper_min, u in res.splits:
        assert lower_max <= upper_min


def test_power_iteration_reaches_top_eigenvector_of_sample_covariance():
    # With many iterations the power iteration converges to the leading
    # eigenvector of the sample covariance (library eigensolver as the check).
    r = rng(9)
    d = 8
    scales = np.array([5.0, 2.0, 1.0, 0.8, 0.6, 0.4, 0.3, 0.2])
    Y = r.standard_normal((256, d)) * scales
    res = orc.pddp_partition(Y, np.eye(d), 64, seed=4, bh=0, tensor=0,
                             power_iters=200, record=True)
    heap, size, t, _, _, u = res.splits[0]
    key = orc.node_key(4, 0, 0, 1)
    pos = orc._sample_positions(256, d, key)
    S = Y[pos] - Y[pos].mean(axis=0)
    lam, U = np.linalg.eigh(S.T @ S / d)
    top = U[:, -1]
    assert min(np.linalg.norm(u - top), np.linalg.norm(u + top)) < 1e-10


@pytest.mark.parametrize("transform", [False, True])
def test_rank_one_data_reduces_to_sorting(transform):
    # Vectors t_i e_1: every principal direction is +-e_1, so every cluster is
    # a run of consecutive ranks of t (textbook sort).
    r = rng(10)
    n, d, c = 1000, 6, 64
    t = r.standard_normal(n)
    X = np.zeros((n, d)); X[:, 0] = t
    Q = r.standard_normal((n, d))
    if transform:
        hc = orc.cluster_head(Q, X, c, seed=5)
        perm, cnt = hc.perm_k, hc.count_k
    else:
        hc = orc.cluster_head(X, X, c, seed=5, transform=False)
        perm, cnt = hc.perm_q, hc.count_q
    rank = np.empty(n, dtype=np.int64); rank[np.argsort(t, kind="stable")] = np.arange(n)
    C = orc.num_clusters(n, c)
    for a in range(C):
        rk = np.sort(rank[perm[a * c: a * c + cnt[a]]])
        assert rk[-1] - rk[0] == cnt[a] - 1


def test_two_cluster_split_is_order_statistic():
    # n = 2c with rank-one data: one cluster holds the c smallest t, the other
    # the c largest (brute force over the sorted values).
    r = rng(11)
    c = 64
    t = r.standard_normal(2 * c)
    X = np.zeros((2 * c, 4)); X[:, 0] = t
    hc = orc.cluster_head(X, X, c, seed=0, transform=False)
    lowest = set(np.argsort(t)[:c].tolist())
    first = set(hc.perm_q[:c].tolist())
    assert first == lowest or first == set(range(2 * c)) - lowest


def test_metric_injected_form_gives_same_partition():
    # Section 6.1: the metric can be injected into the power iteration, so no
    # eigendecomposition is needed. Both forms must give one partition.
    r = rng(12)
    n, d, c = 2048, 16, 64
    Z = r.standard_normal((n, 4))
    Q = Z @ r.standard_normal((4, d)) + 0.1 * r.standard_normal((n, d))
    K = Z @ r.standard_normal((4, d)) + 0.1 * r.standard_normal((n, d))
    M_q, M_k, _ = orc.metric_matrices(Q, K)
    R_q, R_k = orc.psd_root(M_q), orc.psd_root(M_k)
    lit_k = orc.pddp_partition(orc.key_representation(K, R_q), R_q, c, seed=9, bh=0, tensor=1)
    inj_k = orc.pddp_partition_metric_form(K, M_q, c, seed=9, bh=0, tensor=1)
    s = np.sqrt(np.einsum("ij,jk,ik->i", Q, M_k, Q))
    lit_q = orc.pddp_partition(orc.query_representation(Q, R_k), R_k, c, seed=9, bh=0, tensor=0)
    inj_q = orc.pddp_partition_metric_form(Q / s[:, None], M_k, c, seed=9, bh=0, tensor=0)
    for a, b in ((lit_k, inj_k), (lit_q, inj_q)):
        assert len(a.leaves) == len(b.leaves)
        for x, y in zip(a.leaves, b.leaves):
            assert np.array_equal(x, y)


# ---------------------------------------------------------------------------
# Assignment (Section 3.3)
# ---------------------------------------------------------------------------

def test_centroid_score_is_mean_pairwise_logit_eq18():
    r = rng(13)
    Q = r.standard_normal((300, 8)); K = r.standard_normal((300, 8))
    hc = orc.cluster_head(Q, K, 64, seed=2)
    S = orc.centroid_scores(hc.qbar, hc.kbar)
    for a in range(len(hc.count_q)):
        qa = Q[hc.perm_q[a * 64: a * 64 + hc.count_q[a]]]
        for b in range(len(hc.count_k)):
            kb = K[hc.perm_k[b * 64: b * 64 + hc.count_k[b]]]
            brute = sum(float(q @ k) for q in qa for k in kb) / (len(qa) * len(kb))
            assert abs(S[a, b] - brute) < 1e-12


def test_topk_matches_full_sort_with_ties():
    r = rng(14)
    S = np.round(r.standard_normal((40, 57)), 1)    # many exact ties
    k = 9
    kept = orc.topk_route(S, k)
    for a in range(40):
        full = sorted(range(57), key=lambda b: (-S[a, b], b))
        assert list(kept[a]) == sorted(full[:k])
    bits = orc.route_bits(kept, 57)
    for a in range(40):
        got = [b for b in range(57) if (int(bits[a, b // 32]) >> (b % 32)) & 1]
        assert got == list(kept[a])


# ---------------------------------------------------------------------------
# Attention (eq. 1-6, 21-33)
# ---------------------------------------------------------------------------

def _setup_attention(seed=15, n=512, d=16, c=64, random_clusters=False):
    r = rng(seed)
    Q = _mixture(r, n, d); K = _mixture(r, n, d); V = r.standard_normal((n, d))
    if random_clusters:
        C = orc.num_clusters(n, c)
        pq = r.permutation(n); pk = r.permutation(n)
        def to_perm(p):
            perm = np.full(C * c, -1, np.int32); cnt = np.zeros(C, np.int32)
            for a in range(C):
                mem = np.sort(p[a * c:(a + 1) * c]); perm[a * c:a * c + len(mem)] = mem; cnt[a] = len(mem)
            return perm, cnt
        perm_q, count_q = to_perm(pq); perm_k, count_k = to_perm(pk)
        qbar = np.stack([Q[perm_q[a*c:a*c+count_q[a]]].mean(0) for a in range(C)])
        kbar = np.stack([K[perm_k[a*c:a*c+count_k[a]]].mean(0) for a in range(C)])
    else:
        hc = orc.cluster_head(Q, K, c, seed=seed)
        perm_q, count_q, perm_k, count_k = hc.perm_q, hc.count_q, hc.perm_k, hc.count_k
        qbar, kbar = hc.qbar, hc.kbar
    return Q, K, V, perm_q, count_q, perm_k, count_k, qbar, kbar


def test_dense_attention_matches_library_sdpa():
    torch = pytest.importorskip("torch")
    r = rng(16)
    Q = r.standard_normal((200, 32)); K = r.standard_normal((200, 32)); V = r.standard_normal((200, 32))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None])[0].numpy()
    assert np.abs(orc.dense_attention(Q, K, V) - ref).max() < 1e-12


@pytest.mark.parametrize("compensate", [True, False])
def test_keeping_every_cluster_is_dense(compensate):
    Q, K, V, pq, cq, pk, ck, qbar, kbar = _setup_attention(n=500)
    C = len(ck)
    kept = orc.topk_route(orc.centroid_scores(qbar, kbar), C)
    O = orc.compensated_attention(Q, K, V, pq, cq, pk, ck, kept, 64, compensate=compensate)
    assert np.abs(O - orc.dense_attention(Q, K, V)).max() < 1e-12


def test_singleton_clusters_make_compensation_exact():
    # c = 1: every excluded "cluster" is one token whose centroid is the token.
    r = rng(17)
    n, d = 96, 8
    Q = r.standard_normal((n, d)); K = r.standard_normal((n, d)); V = r.standard_normal((n, d))
    perm = np.arange(n, dtype=np.int32); cnt = np.ones(n, np.int32)
    kept = orc.topk_route(orc.centroid_scores(Q, K), 5)
    O = orc.compensated_attention(Q, K, V, perm, cnt, perm, cnt, kept, 1)
    assert np.abs(O - orc.dense_attention(Q, K, V)).max() < 1e-12


def test_cluster_constant_data_makes_compensation_exact_for_every_k():
    # 16 components x 64 identical copies, c = 64: clusters are the components,
    # delta_c = 0 and Cov_c = 0 in eq. 33, so SMC equals dense for every k.
    r = rng(18)
    d, c = 16, 64
    mu_q = r.standard_normal((16, d)); mu_k = r.standard_normal((16, d)); mu_v = r.standard_normal((16, d))
    z = np.repeat(np.arange(16), 64); z = z[r.permutation(z.size)]
    Q, K, V = mu_q[z], mu_k[z], mu_v[z]
    hc = orc.cluster_head(Q, K, c, seed=1)
    for a in range(16):
        assert len(set(z[hc.perm_k[a * c:(a + 1) * c]])) == 1
        assert len(set(z[hc.perm_q[a * c:(a + 1) * c]])) == 1
    dense = orc.dense_attention(Q, K, V)
    S = orc.centroid_scores(hc.qbar, hc.kbar)
    for k in (1, 3, 8, 16):
        kept = orc.topk_route(S, k)
        O = orc.compensated_attention(Q, K, V, hc.perm_q, hc.count_q, hc.perm_k, hc.count_k, kept, c)
        assert np.abs(O - dense).max() < 1e-12


def _brute_weights(q, K, scale):
    lg = np.array([float(q @ k) * scale for k in K])
    e = np.exp(lg - lg.max())
    return e / e.sum(), lg.max(), e.sum()


def test_compensation_error_identity_eq33_and_denominator_eq28():
    # Appendix A. With the dense weights w_i (sum 1) and w_c the centroid
    # weight on the same scale, delta_c = mean_{i in c} w_i - w_c >= 0 and
    #   o - o_hat = (1/d_hat) sum_{c excl} |c| (delta_c (v_bar_c - o) + Cov_c(w, v)),
    #   d_hat - 1 = - sum_{c excl} |c| delta_c.
    Q, K, V, pq, cq, pk, ck, qbar, kbar = _setup_attention(seed=19, n=256, d=8, c=32,
                                                           random_clusters=True)
    c = 32
    d = Q.shape[1]; scale = 1.0 / math.sqrt(d)
    kept = orc.topk_route(orc.centroid_scores(qbar, kbar), 3)
    O_hat = orc.compensated_attention(Q, K, V, pq, cq, pk, ck, kept, c)
    dense = orc.dense_attention(Q, K, V)
    C = len(ck)
    for i in range(0, 256, 17):
        a = int(np.nonzero(pq == i)[0][0]) // c
        w, mx, Z = _brute_weights(Q[i], K, scale)
        o = dense[i]
        excl = [b for b in range(C) if b not in set(kept[a].tolist())]
        w_S = sum(w[j] for b in kept[a] for j in pk[b * c:b * c + ck[b]])
        d_hat = w_S
        rhs = np.zeros(d)
        for b in excl:
            mem = pk[b * c:b * c + ck[b]]
            kb = K[mem].mean(0); vb = V[mem].mean(0)
            w_c = math.exp(float(Q[i] @ kb) * scale - mx) / Z
            wbar = w[mem].mean()
            delta = wbar - w_c
            assert delta >= -1e-15                        # Jensen, eq. 19
            cov = sum((w[j] - wbar) * (V[j] - vb) for j in mem) / len(mem)
            rhs += len(mem) * (delta * (vb - o) + cov)
            d_hat += len(mem) * w_c
        delta_sum = sum(len(pk[b*c:b*c+ck[b]]) * (w[pk[b*c:b*c+ck[b]]].mean()
                        - math.exp(float(Q[i] @ K[pk[b*c:b*c+ck[b]]].mean(0)) * scale - mx) / Z)
                        for b in excl)
        assert abs((d_hat - 1.0) + delta_sum) < 1e-12      # eq. 28
        assert np.abs((o - O_hat[i]) - rhs / d_hat).max() < 1e-12   # eq. 33


def test_uncompensated_error_identity_eq4():
    # eq. 3-4: o - o_S = (1 - w_S)(o_Sbar - o_S).
    Q, K, V, pq, cq, pk, ck, qbar, kbar = _setup_attention(seed=20, n=256, d=8, c=32)
    c = 32; scale = 1.0 / math.sqrt(8)
    kept = orc.topk_route(orc.centroid_scores(qbar, kbar), 2)
    O_S = orc.compensated_attention(Q, K, V, pq, cq, pk, ck, kept, c, compensate=False)
    dense = orc.dense_attention(Q, K, V)
    for i in range(0, 256, 13):
        a = int(np.nonzero(pq == i)[0][0]) // c
        w, _, _ = _brute_weights(Q[i], K, scale)
        S = np.concatenate([pk[b * c:b * c + ck[b]] for b in kept[a]])
        Sbar = np.setdiff1d(np.arange(256), S)
        w_S = w[S].sum()
        o_Sbar = (w[Sbar, None] * V[Sbar]).sum(0) / w[Sbar].sum()
        assert np.abs((dense[i] - O_S[i]) - (1 - w_S) * (o_Sbar - O_S[i])).max() < 1e-12


def test_compensation_error_shrinks_as_clusters_tighten():
    # Section 1.2 / Appendix A: both terms of eq. 33 shrink with tighter
    # clusters. 16 components x 64 tokens, labels shared by Q, K and V,
    # per-component spread sigma; mean error over 8 seeds must fall with sigma
    # and vanish at sigma = 0.
    d, c, k = 16, 64, 4
    errs = []
    for sigma in (0.3, 0.1, 0.03, 0.0):
        e = []
        for seed in range(8):
            r = rng(100 + seed)
            mq, mk, mv = (r.standard_normal((16, d)) for _ in range(3))
            z = np.repeat(np.arange(16), 64); z = z[r.permutation(z.size)]
            Q = mq[z] + sigma * r.standard_normal((1024, d))
            K = mk[z] + sigma * r.standard_normal((1024, d))
            V = mv[z] + sigma * r.standard_normal((1024, d))
            fr = orc.forward_head(Q, K, V, c, k, seed=seed)
            e.append(np.abs(fr.O - orc.dense_attention(Q, K, V)).mean())
        errs.append(float(np.mean(e)))
    assert errs[0] > errs[1] > errs[2] > errs[3]
    assert errs[3] < 1e-12


# ---------------------------------------------------------------------------
# Adaptive selection (Section 3.3.2 "Selection") and the adaptive query
# representation (eq. 15)
# ---------------------------------------------------------------------------

def _brute_adaptive(scores, count_k, d, recall, min_count):
    """Direct evaluation of the definition: sort by mass with Python's sort,
    add masses one at a time with math.fsum-free plain floats in that order."""
    Cq, Ck = scores.shape
    out = []
    for a in range(Cq):
        w = [float(scores[a, b]) / math.sqrt(d) + math.log(float(count_k[b])) for b in range(Ck)]
        order = sorted(range(Ck), key=lambda b: (-w[b], b))
        mass = [math.exp(w[b] - w[order[0]]) for b in order]
        total = 0.0
        for m in mass:
            total += m
        cum, k = 0.0, Ck
        for i, m in enumerate(mass):
            cum += m
            if cum >= recall * total:
                k = i + 1
                break
        if recall <= 0:
            k = 1
        k = max(k, min(min_count, Ck))
        out.append(sorted(order[:k]))
    return out


@pytest.mark.parametrize("recall", [0.0, 0.3, 0.9, 0.999, 1.0])
def test_adaptive_route_matches_brute_force(recall):
    r = rng(31)
    d = 16
    scores = r.normal(size=(12, 40)) * 4.0
    count_k = r.integers(1, 200, size=40)
    got = orc.adaptive_route(scores, count_k, d, recall, min_count=5)
    want = _brute_adaptive(scores, count_k, d, recall, 5)
    assert [list(g) for g in got] == want


def test_adaptive_route_at_zero_recall_is_top_k_by_mass():
    # The paper: for top-k assignment the recall threshold is 0, so the count
    # threshold alone decides; with equal counts the mass order is the score
    # order and the result is exactly top-k.
    r = rng(32)
    scores = r.normal(size=(9, 30))
    count_k = np.full(30, 64)
    got = orc.adaptive_route(scores, count_k, 64, 0.0, min_count=7)
    want = orc.topk_route(scores, 7)
    assert all(np.array_equal(g, w) for g, w in zip(got, want))


def test_adaptive_route_weights_cluster_size():
    # Two clusters, the second with a lower centroid score but 1000 times the
    # members: its estimated mass |b| e^{s/sqrt(d)} is larger, so it is taken
    # first and alone reaches a 50% recall.
    d = 4
    scores = np.array([[2.0, 0.0]])
    count_k = np.array([1, 1000])
    got = orc.adaptive_route(scores, count_k, d, 0.5, min_count=1)
    assert list(got[0]) == [1]


def test_adaptive_route_is_minimal_and_reaches_recall():
    r = rng(33)
    d = 32
    scores = r.normal(size=(20, 64)) * 6.0
    count_k = r.integers(50, 130, size=64)
    recall = 0.8
    W = scores / math.sqrt(d) + np.log(count_k)[None, :]
    for a, kept in enumerate(orc.adaptive_route(scores, count_k, d, recall, min_count=3)):
        m = np.exp(W[a] - W[a].max())
        total = m.sum()
        assert m[kept].sum() >= recall * total * (1 - 1e-12)
        if len(kept) > 3:
            # dropping the lightest kept cluster falls below the recall
            lightest = kept[np.argmin(m[kept])]
            assert m[kept].sum() - m[lightest] < recall * total
        # every kept cluster outweighs every excluded one
        excl = np.setdiff1d(np.arange(64), kept)
        assert m[kept].min() >= m[excl].max()


def test_adaptive_query_representation_is_the_eq15_metric():
    # |R_k (q1 - q2)|^2 = (q1 - q2)^T K_c^T K_c (q1 - q2) / n (eq. 15).
    r = rng(34)
    Q = r.normal(size=(200, 8)); K = r.normal(size=(200, 8)) + 0.5   # n tokens of each
    _, M_k, _ = orc.metric_matrices(Q, K)
    Kc = K - K.mean(axis=0)
    Y = orc.query_representation_adaptive(Q, orc.psd_root(M_k))
    for i, j in [(0, 1), (3, 17), (20, 49)]:
        dq = Q[i] - Q[j]
        want = float(np.sum((Kc @ dq) ** 2)) / K.shape[0]
        got = float(np.sum((Y[i] - Y[j]) ** 2))
        assert got == pytest.approx(want, rel=1e-10)


def test_adaptive_route_breaks_mass_ties_to_the_lower_index():
    # Equal scores and counts: every cluster has the same mass, so the first
    # min_count clusters (lowest indices) are kept, and with 50% recall of 10
    # equal masses, exactly the first 5.
    scores = np.zeros((2, 10))
    count_k = np.full(10, 32)
    got = orc.adaptive_route(scores, count_k, 16, 0.0, min_count=3)
    assert [list(g) for g in got] == [[0, 1, 2], [0, 1, 2]]
    got = orc.adaptive_route(scores, count_k, 16, 0.5, min_count=1)
    assert list(got[0]) == [0, 1, 2, 3, 4]


# ---------------------------------------------------------------------------
# Random-cluster baseline (the paper's error analysis compares the recursive
# split with random clusters)
# ---------------------------------------------------------------------------

def test_random_leaves_partition_and_sizes():
    n, c = 1000, 64
    leaves = orc.random_leaves(n, c, seed=3, bh=1, tensor=0)
    sizes = [len(l) for l in leaves]
    assert sizes == [c] * (n // c) + [n % c]        # remainder last, as in the split tree
    allm = np.concatenate(leaves)
    assert np.array_equal(np.sort(allm), np.arange(n))
    assert all(np.all(np.diff(l) > 0) for l in leaves)


def test_random_leaves_follow_the_splitmix_keys():
    # brute force: the first group holds the c tokens with the smallest keys
    n, c = 300, 32
    base = orc.node_key(9, 0, 1, 0)
    keys = [orc.splitmix64(base ^ i) for i in range(n)]
    first = sorted(sorted(range(n), key=lambda i: (keys[i], i))[:c])
    assert list(orc.random_leaves(n, c, seed=9, bh=0, tensor=1)[0]) == first


def test_tight_clusters_beat_random_ones_when_attention_is_sparse_and_with_compensation():
    # The paper's error analysis (Section 1.2 / 3): when the sparsity
    # assumption holds (well-separated mixture components, values independent
    # of keys), tight clusters that capture the attention mass give the
    # smaller error; and with centroid compensation tighter clusters give the
    # smaller error in any case. Random clusters are the paper's baseline.
    import workloads as wl
    w = wl.make_workload("mixture", H=1, N=1024, d=32, c=32, k=4, dtype="fp32", seed=40)
    Qf, Kf, Vf = (x[0, 0].astype(np.float64) for x in (w.Q, w.K, w.V))
    dense = orc.dense_attention(Qf, Kf, Vf)
    err = {}
    for name, h in (("split", orc.cluster_head(Qf, Kf, w.c, seed=0)),
                    ("random", orc.cluster_head_random(Qf, Kf, w.c, seed=0))):
        kept = orc.topk_route(orc.centroid_scores(h.qbar, h.kbar), w.k)
        for comp in (False, True):
            O = orc.compensated_attention(Qf, Kf, Vf, h.perm_q, h.count_q, h.perm_k, h.count_k, kept, w.c,
                                          compensate=comp)
            err[name, comp] = np.linalg.norm(O - dense) / np.linalg.norm(dense)
    assert err["split", False] < err["random", False]
    assert err["split", True] < err["random", True]


# ---------------------------------------------------------------------------
# Diagonalized recursive splitting (Section 3.2.1 "Diagonalized recursive
# splitting"; later revision Section 4.1.1).
# ---------------------------------------------------------------------------

def test_pca_basis_matches_svd_of_centred_rows():
    """The basis diagonalises the covariance: compare with the right singular
    vectors of the centred rows (a different library routine), eigenvalue =
    singular value^2 / n, same order, same sign rule."""
    rng = np.random.default_rng(101)
    A = rng.standard_normal((6, 6))
    Y = rng.standard_normal((400, 6)) @ A + rng.standard_normal(6) * 3.0
    U, lam = orc.pca_basis(Y)
    Yc = Y - Y.mean(axis=0)
    _, sv, Vt = np.linalg.svd(Yc, full_matrices=False)
    np.testing.assert_allclose(lam, sv ** 2 / Y.shape[0], rtol=1e-12)
    assert np.all(np.diff(lam) <= 0)
    for j in range(6):
        v = Vt[j]
        i = int(np.argmax(np.abs(v)))
        v = v if v[i] > 0 else -v
        np.testing.assert_allclose(U[:, j], v, atol=1e-10)
        assert U[np.argmax(np.abs(U[:, j])), j] > 0


def test_diagonal_split_of_line_data_follows_the_signed_principal_direction():
    """Points along a known direction u (largest entry positive) plus small
    noise: the first split puts the t points with the smallest u . y below it,
    whatever their token order."""
    rng = np.random.default_rng(102)
    d, n, c = 8, 200, 16
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    if u[np.argmax(np.abs(u))] < 0:
        u = -u
    s = rng.standard_normal(n) * 10.0
    Y = s[:, None] * u[None, :] + rng.standard_normal((n, d)) * 1e-3
    r = orc.diagonal_partition(Y, c, seed=0, bh=0, tensor=0, record=True)
    heap, size, t, lo_max, up_min, j = r.splits[0]
    assert heap == 1 and size == n and j == 0      # the leading coordinate
    t_want = orc.split_count(n, c)
    assert t == t_want and t != n - t
    below = np.sort(np.argsort(Y @ u, kind="stable")[:t])
    # leaves of the left subtree are exactly the t smallest along +u
    left = np.sort(np.concatenate([lv for lv in r.leaves if np.isin(lv, below).all()]))
    np.testing.assert_array_equal(left, below)


def test_diagonal_root_split_uses_leading_component_when_sample_is_whole_set():
    """With |S| <= d the sample is the whole set, whose variance along basis
    vector j is eigenvalue j: the root splits on the leading principal
    component (a flipped eigenvalue order would pick the smallest)."""
    rng = np.random.default_rng(103)
    d, n, c = 32, 32, 4
    Y = rng.standard_normal((n, d)) * np.linspace(3.0, 0.1, d)
    r = orc.diagonal_partition(Y, c, seed=5, bh=1, tensor=1, record=True)
    _, _, t, _, _, j = r.splits[0]
    assert j == 0
    Yc = Y - Y.mean(axis=0)
    _, _, Vt = np.linalg.svd(Yc, full_matrices=False)
    v = Vt[0] if Vt[0][np.argmax(np.abs(Vt[0]))] > 0 else -Vt[0]
    proj = Y @ v
    below = set(np.lexsort((np.arange(n), proj))[:t].tolist())
    first_leaves = []
    acc = 0
    for lv in r.leaves:
        if acc >= t:
            break
        first_leaves.extend(lv.tolist())
        acc += len(lv)
    assert set(first_leaves) == below


def test_diagonal_partition_invariant_to_coordinate_permutation():
    """Permuting the coordinates of every row permutes the basis vectors'
    entries (largest entry and its sign kept): the same partition."""
    rng = np.random.default_rng(104)
    d, n, c = 12, 900, 32
    A = rng.standard_normal((d, d))
    Y = rng.standard_normal((n, d)) @ A
    pi = rng.permutation(d)
    r1 = orc.diagonal_partition(Y, c, seed=3, bh=0, tensor=0)
    r2 = orc.diagonal_partition(Y[:, pi], c, seed=3, bh=0, tensor=0)
    assert r1.min_margin > 1e-9
    assert len(r1.leaves) == len(r2.leaves)
    for a, b in zip(r1.leaves, r2.leaves):
        np.testing.assert_array_equal(a, b)


def test_diagonal_partition_of_sign_symmetric_data_is_coordinate_splitting():
    """Rows made of every sign pattern of a few base rows have an exactly
    diagonal covariance, so the basis is the coordinate axes sorted by
    variance (the sign rule makes each axis +e_i) and every split is a split
    on the raw coordinate of highest sample variance: checked against that
    direct procedure."""
    rng = np.random.default_rng(105)
    d, c = 3, 8
    base = rng.uniform(0.5, 1.5, size=(13, d)) * np.array([2.0, 1.0, 3.0])
    signs = np.array([[1 if (m >> b) & 1 else -1 for b in range(d)] for m in range(2 ** d)])
    Y = (base[:, None, :] * signs[None, :, :]).reshape(-1, d)
    n = Y.shape[0]
    r = orc.diagonal_partition(Y, c, seed=9, bh=2, tensor=1, sample_factor=4)

    want = []

    def rec(members, heap):
        if members.shape[0] <= c:
            want.append(members)
            return
        size = members.shape[0]
        key = orc.node_key(9, 2, 1, heap)
        m = min(4 * d, size)
        if size <= m:
            pos = np.arange(size)
        else:
            off = orc.sample_offset(key, size)
            pos = (np.arange(m) * size + off) // m
        S = Y[members[pos]]
        j = int(np.argmax(S.var(axis=0)))
        t = orc.split_count(size, c)
        order = np.lexsort((members, Y[members, j]))
        rec(np.sort(members[order[:t]]), 2 * heap)
        rec(np.sort(members[order[t:]]), 2 * heap + 1)

    rec(np.arange(n), 1)
    assert len(r.leaves) == len(want)
    for a, b in zip(r.leaves, want):
        np.testing.assert_array_equal(a, b)


def test_diagonal_cluster_head_partitions_both_tensors():
    rng = np.random.default_rng(106)
    n, d, c = 1000, 16, 64
    Q = rng.standard_normal((n, d))
    K = rng.standard_normal((n, d)) + 0.5
    for transform in (True, False):
        for form in ("topk", "adaptive"):
            h = orc.cluster_head(Q, K, c, seed=1, transform=transform, query_form=form,
                                 splitting="diagonal")
            for perm, cnt in ((h.perm_q, h.count_q), (h.perm_k, h.count_k)):
                assert sorted(perm[perm >= 0].tolist()) == list(range(n))
                assert cnt.sum() == n and (cnt[:-1] == c).all()


def test_diagonal_partition_does_not_depend_on_the_metric_factor():
    """Any factor F with F F^T = M gives the representation X F a rotation of
    X R (R the symmetric root), whose principal coordinates are the same up
    to sign; the sign rule is stated on the raw-space direction F u_j, so
    the partition with the symmetric root and with the Cholesky factor (a
    different library routine) is the same."""
    rng = np.random.default_rng(107)
    n, d, c = 1500, 12, 64
    X = rng.standard_normal((n, d)) @ rng.standard_normal((d, d)) + 0.3
    Qm = rng.standard_normal((3 * n, d)) @ rng.standard_normal((d, d))
    M = Qm.T @ Qm / Qm.shape[0]
    R = orc.psd_root(M)
    L = np.linalg.cholesky(M)
    np.testing.assert_allclose(L @ L.T, R @ R, rtol=1e-10, atol=1e-10)
    for seed in range(4):
        r1 = orc.diagonal_partition(X @ R, c, seed=seed, bh=0, tensor=1, factor=R)
        r2 = orc.diagonal_partition(X @ L, c, seed=seed, bh=0, tensor=1, factor=L)
        assert r1.min_margin > 1e-9
        for a, b in zip(r1.leaves, r2.leaves):
            np.testing.assert_array_equal(a, b)
    # the raw-space directions themselves agree, signs included
    U_r, _ = orc.pca_basis(X @ R, R)
    U_l, _ = orc.pca_basis(X @ L, L)
    np.testing.assert_allclose(R @ U_r, L @ U_l, atol=1e-8)


# ---------------------------------------------------------------------------
# Unequal query and key cluster sizes (the paper evaluates 64 for queries and
# 128 for keys, Section 3.1).
# ---------------------------------------------------------------------------

def test_unequal_cluster_sizes_follow_each_tensors_tree():
    r = rng(108)
    n, d = 1000, 16
    Q = r.standard_normal((n, d)); K = r.standard_normal((n, d))
    hc = orc.cluster_head(Q, K, 64, seed=2, c_k=128)
    assert hc.count_q.tolist() == [64] * 15 + [40]
    assert hc.count_k.tolist() == [128] * 7 + [104]
    assert hc.perm_q.shape[0] == 16 * 64 and hc.perm_k.shape[0] == 8 * 128
    for perm in (hc.perm_q, hc.perm_k):
        assert sorted(perm[perm >= 0].tolist()) == list(range(n))
    # equal sizes through c_k give the default call exactly
    a = orc.cluster_head(Q, K, 64, seed=2)
    b = orc.cluster_head(Q, K, 64, seed=2, c_k=64)
    np.testing.assert_array_equal(a.perm_k, b.perm_k)
    np.testing.assert_array_equal(a.perm_q, b.perm_q)


@pytest.mark.parametrize("compensate", [True, False])
def test_unequal_sizes_keeping_every_key_cluster_is_dense(compensate):
    r = rng(109)
    n, d = 700, 16
    Q = r.standard_normal((n, d)); K = r.standard_normal((n, d)); V = r.standard_normal((n, d))
    hc = orc.cluster_head(Q, K, 64, seed=3, c_k=128)
    S = orc.centroid_scores(hc.qbar, hc.kbar)
    assert S.shape == (11, 6)
    kept = orc.topk_route(S, 6)
    O = orc.compensated_attention(Q, K, V, hc.perm_q, hc.count_q, hc.perm_k, hc.count_k, kept, 64,
                                  compensate=compensate, c_k=128)
    assert np.abs(O - orc.dense_attention(Q, K, V)).max() < 1e-12


def test_unequal_sizes_cluster_constant_keys_make_compensation_exact():
    # 8 key components x 128 identical keys (and values), queries free: with
    # c_k = 128 the key clusters are the components, so every excluded key
    # cluster is represented exactly by |b| e^{q . k_bar / sqrt(d)} v_bar, for
    # every k, while the queries are split at c_q = 64.
    r = rng(110)
    d = 16
    mu_k = r.standard_normal((8, d)); mu_v = r.standard_normal((8, d))
    z = np.repeat(np.arange(8), 128); z = z[r.permutation(z.size)]
    K, V = mu_k[z], mu_v[z]
    Q = r.standard_normal((z.size, d))
    hc = orc.cluster_head(Q, K, 64, seed=4, c_k=128)
    for b in range(8):
        assert len(set(z[hc.perm_k[b * 128:(b + 1) * 128]])) == 1
    assert hc.count_q.tolist() == [64] * 16
    dense = orc.dense_attention(Q, K, V)
    S = orc.centroid_scores(hc.qbar, hc.kbar)
    for k in (1, 3, 8):
        kept = orc.topk_route(S, k)
        O = orc.compensated_attention(Q, K, V, hc.perm_q, hc.count_q, hc.perm_k, hc.count_k, kept, 64, c_k=128)
        assert np.abs(O - dense).max() < 1e-12
        # the key slots read with the query size would be wrong
        if k < 8:
            bad = orc.compensated_attention(Q, K, V, hc.perm_q, hc.count_q, hc.perm_k, hc.count_k, kept, 64)
            assert np.abs(bad - dense).max() > 1e-3
