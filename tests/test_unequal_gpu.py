"""Unequal query and key cluster sizes on the GPU (the paper's evaluated
block shape, Section 3.1 "Overview": 64 queries against 128 keys).

Queries split into clusters of c, keys into clusters of c_k (each tensor
walks its own split tree); routing scores C_q x C_k centroid pairs; the
attention runs c-query tiles against c_k-key clusters. Checked against the
oracle's cluster_head / compensated_attention / forward_head with c_k:
partitions and masks bit-exact, outputs within 1e-2 (bf16) / 1e-5 (fp32).
"""
import numpy as np
import pytest

import workloads as wl
from oracle import ca_oracle as orc

from tests import parity

pytestmark = pytest.mark.gpu

CASES = {
    "q64-k128-bf16-d64": (lambda: wl.make_workload("lowrank", H=2, N=4096, n_valid=4000, d=64, c=64, k=5,
                                                   dtype="bf16", seed=91), 128),
    "q128-k64-bf16-d128": (lambda: wl.make_workload("grid", H=2, N=2048, d=128, c=128, k=6, dtype="bf16", seed=92,
                                                    grid=(8, 16, 16)), 64),
    "q128-k256-bf16-d64": (lambda: wl.make_workload("heavytail", H=1, N=8192, d=64, c=128, k=3, dtype="bf16",
                                                    seed=93), 256),
    "q256-k128-bf16-d64": (lambda: wl.make_workload("mixture", H=2, N=3000, d=64, c=256, k=4, dtype="bf16",
                                                    seed=94), 128),
    "q64-k128-fp32-d64": (lambda: wl.make_workload("mixture", H=1, N=1000, d=64, c=64, k=3, dtype="fp32",
                                                   seed=95), 128),
    "q64-k256-bf16-n2ck+1": (lambda: wl.make_workload("lowrank", H=1, N=640, n_valid=513, d=64, c=64, k=2,
                                                      dtype="bf16", seed=96), 256),
}


@pytest.fixture(scope="module")
def helpers():
    from tests import gpu_helpers
    return gpu_helpers


def _oracle(w, ck):
    return orc.cluster_workload(w.Q.astype(np.float64), w.K.astype(np.float64), w.n_valid, w.c, seed=0, c_k=ck)


@pytest.mark.parametrize("name", list(CASES))
def test_partitions_bit_exact(helpers, name):
    make, ck = CASES[name]
    w = make()
    run = helpers.Run(w, c_k=ck)
    assert run.Ck == orc.num_clusters(w.n_valid, ck)
    got = run.cluster()
    for bh, h in enumerate(_oracle(w, ck)):
        np.testing.assert_array_equal(got["count_q"][bh], h.count_q)
        np.testing.assert_array_equal(got["count_k"][bh], h.count_k)
        np.testing.assert_array_equal(got["perm_q"][bh], h.perm_q, err_msg=f"{name} bh={bh} queries")
        np.testing.assert_array_equal(got["perm_k"][bh], h.perm_k, err_msg=f"{name} bh={bh} keys")
        assert np.abs(got["qbar"][bh] - h.qbar).max() <= 1e-12 * max(1.0, np.abs(h.qbar).max())
        assert np.abs(got["kbar"][bh] - h.kbar).max() <= 1e-12 * max(1.0, np.abs(h.kbar).max())


@pytest.mark.parametrize("name", list(CASES))
def test_routes_bit_exact_given_oracle_centroids(helpers, name):
    make, ck = CASES[name]
    w = make()
    run = helpers.Run(w, c_k=ck)
    ref = _oracle(w, ck)
    run.set_clusters(ref)
    kept, bits = run.route()
    for bh, h in enumerate(ref):
        want = orc.topk_route(orc.centroid_scores(h.qbar, h.kbar), run.k)
        np.testing.assert_array_equal(kept[bh], want)
        np.testing.assert_array_equal(bits[bh], orc.route_bits(want, run.Ck))


@pytest.mark.parametrize("compensate", [True, False])
@pytest.mark.parametrize("name", list(CASES))
def test_attention_given_oracle_clusters_and_mask(helpers, name, compensate):
    make, ck = CASES[name]
    w = make()
    run = helpers.Run(w, c_k=ck, compensate=compensate)
    ref = _oracle(w, ck)
    kept = [orc.topk_route(orc.centroid_scores(h.qbar, h.kbar), run.k) for h in ref]
    run.set_clusters(ref)
    run.set_routes(kept)
    O = run.attend()
    for bh, h in enumerate(ref):
        b, hh = divmod(bh, w.H)
        Qf, Kf, Vf = (x[b, hh, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
        want = orc.compensated_attention(Qf, Kf, Vf, h.perm_q, h.count_q, h.perm_k, h.count_k, kept[bh], w.c,
                                         compensate=compensate, c_k=ck)
        parity.check(f"unequal attend {name} smc={int(compensate)} bh={bh}", O[b, hh, :w.n_valid], want, w.dtype)
        assert np.all(O[b, hh, w.n_valid:] == 0)


@pytest.mark.parametrize("name", ["q64-k128-bf16-d64", "q128-k64-bf16-d128", "q64-k128-fp32-d64"])
def test_forward_end_to_end(helpers, name):
    make, ck = CASES[name]
    w = make()
    run = helpers.Run(w, c_k=ck)
    O = run.forward()
    for bh in range(w.B * w.H):
        b, hh = divmod(bh, w.H)
        Qf, Kf, Vf = (x[b, hh, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
        fr = orc.forward_head(Qf, Kf, Vf, w.c, w.k, seed=0, bh=bh, c_k=ck)
        parity.check(f"unequal forward {name} bh={bh}", O[b, hh, :w.n_valid], fr.O, w.dtype)


def test_adaptive_selection_with_unequal_sizes(helpers):
    make, ck = CASES["q64-k128-bf16-d64"]
    w = make()
    Ck = orc.num_clusters(w.n_valid, ck)
    run = helpers.Run(w, c_k=ck, k=Ck, selection="adaptive", recall=0.8, min_count=4)
    ref = orc.cluster_workload(w.Q.astype(np.float64), w.K.astype(np.float64), w.n_valid, w.c, seed=0, c_k=ck,
                               query_form="adaptive")
    run.set_clusters(ref)
    kept, _ = run.route()
    counts = run.route_counts()
    for bh, h in enumerate(ref):
        want = orc.adaptive_route(orc.centroid_scores(h.qbar, h.kbar), h.count_k, w.d, 0.8, 4)
        for a in range(run.C):
            np.testing.assert_array_equal(kept[bh, a, :counts[bh, a]], want[a])
