"""Adaptive selection and the eq. 15 query representation on the GPU vs the
fp64 oracle ("ClusterAttention", Section 3.3.2 "Selection", second method;
Section 3.2.2 "Query clustering", eq. 15).

Bar: the kept sets equal the oracle's given the oracle's centroids; where the
running mass lands within 1e-12 (relative) of the recall threshold, or two
masses tie within 1e-12, the two sides may round the fp64 exponentials and
sums differently, and the GPU's set is checked to be a valid and minimal
greedy selection instead (a prefix of the mass order up to 1e-12 ties,
reaching the recall target and the minimum count, and not reaching the target
without its lightest member).
Attention with per-cluster kept counts: the same tolerance as top-k.
"""
import math

import numpy as np
import pytest

import workloads as wl
from oracle import ca_oracle as orc

from tests import parity, selection

pytestmark = pytest.mark.gpu

CASES = {
    "lowrank-bf16-d64-n3900pad-c128": lambda: wl.make_workload("lowrank", H=2, N=4096, n_valid=3900, d=64, c=128,
                                                               k=6, dtype="bf16", seed=21),
    "mix-fp32-d64-n1000-c64": lambda: wl.make_workload("mixture", H=2, N=1000, d=64, c=64, k=5, dtype="fp32",
                                                       seed=22),
    "grid-bf16-d128-c128": lambda: wl.make_workload("grid", H=1, N=6144, d=128, c=128, k=7, dtype="bf16", seed=23,
                                                    grid=(8, 9, 80)),
    "heavytail-bf16-d64-c64": lambda: wl.make_workload("heavytail", H=1, N=8192, d=64, c=64, k=8, dtype="bf16",
                                                       seed=24),
}


def _oracle(w, query_form="topk"):
    return orc.cluster_workload(w.Q.astype(np.float64), w.K.astype(np.float64), w.n_valid, w.c, seed=0) \
        if query_form == "topk" else [
            orc.cluster_head(w.Q[b, h, :w.n_valid].astype(np.float64), w.K[b, h, :w.n_valid].astype(np.float64),
                             w.c, seed=0, bh=b * w.H + h, query_form="adaptive")
            for b in range(w.B) for h in range(w.H)]


def _check_set(got, want, W, recall, min_count):
    """Exact equality, or (at a numerical boundary) a valid selection."""
    if np.array_equal(np.sort(got), want):
        return
    m = np.exp(W - W.max())
    order = np.lexsort((np.arange(W.size), -W))
    cum = np.cumsum(m[order])
    k = len(want)
    near_threshold = recall > 0 and abs(cum[k - 1] - recall * cum[-1]) <= 1e-12 * cum[-1] or \
        (k >= 2 and abs(cum[k - 2] - recall * cum[-1]) <= 1e-12 * cum[-1])
    near_tie = abs(len(got) - k) <= 1 and np.any(np.isclose(W[np.setxor1d(got, want)][:, None],
                                                            W[np.setxor1d(got, want)][None, :], rtol=0,
                                                            atol=1e-12 * max(1.0, abs(W).max())) &
                                                 ~np.eye(len(np.setxor1d(got, want)), dtype=bool))
    assert near_threshold or near_tie, f"kept {sorted(got)} vs oracle {list(want)}"
    problem = selection.adaptive_selection_problem(got, W, recall, min_count)
    assert problem is None, problem


@pytest.mark.parametrize("recall", [0.5, 0.9, 0.99])
@pytest.mark.parametrize("name", list(CASES))
def test_adaptive_route_given_oracle_centroids(name, recall):
    from tests import gpu_helpers as gh
    w = CASES[name]()
    C = orc.num_clusters(w.n_valid, w.c)
    min_count = min(16, max(1, C // 4))
    run = gh.Run(w, k=C, selection="adaptive", recall=recall, min_count=min_count)
    ref = _oracle(w)
    run.set_clusters(ref)
    kept, bits = run.route()
    counts = run.route_counts()
    for bh, h in enumerate(ref):
        scores = orc.centroid_scores(h.qbar, h.kbar)
        want = orc.adaptive_route(scores, h.count_k, w.d, recall, min_count)
        Wl = orc.cluster_log_mass(scores, h.count_k, w.d)
        for a in range(C):
            got = kept[bh, a, :counts[bh, a]]
            assert np.all(np.diff(got) > 0), "kept list ascending"
            _check_set(got, want[a], Wl[a], recall, min_count)
            gb = np.zeros(C, bool)
            for b in got:
                gb[b] = True
            words = bits[bh, a]
            unpacked = np.array([(words[b // 32] >> (b % 32)) & 1 for b in range(C)], bool)
            np.testing.assert_array_equal(unpacked, gb)


@pytest.mark.parametrize("compensate", [True, False])
@pytest.mark.parametrize("name", list(CASES))
def test_attend_with_adaptive_counts(name, compensate):
    # attention over variable kept lists (the GPU's own adaptive selection on
    # the oracle's clusters), against the oracle's attention on the same lists
    from tests import gpu_helpers as gh
    w = CASES[name]()
    C = orc.num_clusters(w.n_valid, w.c)
    run = gh.Run(w, k=C, compensate=compensate, selection="adaptive", recall=0.8, min_count=min(4, C))
    ref = _oracle(w)
    run.set_clusters(ref)
    kept, _ = run.route()
    counts = run.route_counts()
    O = run.attend()
    for bh, h in enumerate(ref):
        b, hh = divmod(bh, w.H)
        lists = [kept[bh, a, :counts[bh, a]] for a in range(C)]
        Qf, Kf, Vf = (x[b, hh, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
        want = orc.compensated_attention(Qf, Kf, Vf, h.perm_q, h.count_q, h.perm_k, h.count_k, lists, w.c,
                                         compensate=compensate)
        parity.check(f"adaptive {name} bh={bh}", O[b, hh, :w.n_valid], want, w.dtype)
        assert counts[bh].min() >= 1 and counts[bh].max() <= C


@pytest.mark.parametrize("name", list(CASES))
def test_adaptive_query_form_partition_bit_exact(name):
    from tests import gpu_helpers as gh
    w = CASES[name]()
    C = orc.num_clusters(w.n_valid, w.c)
    run = gh.Run(w, k=C, selection="adaptive")
    got = run.cluster()
    ref = _oracle(w, "adaptive")
    for bh, h in enumerate(ref):
        np.testing.assert_array_equal(got["perm_q"][bh], h.perm_q, err_msg=f"{name} bh={bh}, oracle min split "
                                      f"margin {h.min_margin_q:.3g}")
        np.testing.assert_array_equal(got["perm_k"][bh], h.perm_k)
