"""GPU path vs the fp64 oracle, element by element, through the C ABI.

Bar:
 * cluster sizes and the partition: bit-exact;
 * routing masks: bit-exact given the oracle's centroids;
 * attention output given the oracle's permutation, mask and centroids:
   max-abs error <= 1e-2 for bf16 inputs (bf16 products, fp32 accumulation),
   <= 1e-5 for fp32 inputs, and relative-L2 error within the bounds derived
   in tests/parity.py (observed values printed at the end of the session).
"""
import math

import numpy as np
import pytest

import workloads as wl
from oracle import ca_oracle as orc

from tests import parity
from tests.cases import CASES

pytestmark = pytest.mark.gpu

TOL = parity.MAX_ABS


def oracle_clusters(w, seed=0):
    return orc.cluster_workload(w.Q.astype(np.float64), w.K.astype(np.float64), w.n_valid, w.c, seed=seed)


@pytest.fixture(scope="module")
def helpers():
    from tests import gpu_helpers
    return gpu_helpers


@pytest.mark.parametrize("name", list(CASES))
def test_cluster_partition_bit_exact(helpers, name):
    w = CASES[name]()
    run = helpers.Run(w)
    got = run.cluster()
    ref = oracle_clusters(w)
    for bh, h in enumerate(ref):
        np.testing.assert_array_equal(got["count_q"][bh], h.count_q)
        np.testing.assert_array_equal(got["count_k"][bh], h.count_k)
        np.testing.assert_array_equal(got["perm_q"][bh], h.perm_q, err_msg=f"{name} bh={bh} queries, "
                                      f"oracle min split margin {h.min_margin_q:.3g}")
        np.testing.assert_array_equal(got["perm_k"][bh], h.perm_k, err_msg=f"{name} bh={bh} keys, "
                                      f"oracle min split margin {h.min_margin_k:.3g}")
        assert np.abs(got["qbar"][bh] - h.qbar).max() <= 1e-12 * max(1.0, np.abs(h.qbar).max())
        assert np.abs(got["kbar"][bh] - h.kbar).max() <= 1e-12 * max(1.0, np.abs(h.kbar).max())


@pytest.mark.parametrize("name", list(CASES))
def test_route_bit_exact_given_oracle_centroids(helpers, name):
    w = CASES[name]()
    run = helpers.Run(w)
    ref = oracle_clusters(w)
    run.set_clusters(ref)
    kept, bits = run.route()
    for bh, h in enumerate(ref):
        want = orc.topk_route(orc.centroid_scores(h.qbar, h.kbar), run.k)
        np.testing.assert_array_equal(kept[bh], want)
        np.testing.assert_array_equal(bits[bh], orc.route_bits(want, run.C))


@pytest.mark.parametrize("compensate", [True, False])
@pytest.mark.parametrize("name", list(CASES))
def test_attend_given_oracle_clusters_and_mask(helpers, name, compensate):
    w = CASES[name]()
    run = helpers.Run(w, compensate=compensate)
    ref = oracle_clusters(w)
    kept = [orc.topk_route(orc.centroid_scores(h.qbar, h.kbar), run.k) for h in ref]
    run.set_clusters(ref)
    run.set_routes(kept)
    O = run.attend()
    for bh, h in enumerate(ref):
        b, hh = divmod(bh, w.H)
        Qf, Kf, Vf = (x[b, hh, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
        want = orc.compensated_attention(Qf, Kf, Vf, h.perm_q, h.count_q, h.perm_k, h.count_k, kept[bh], w.c,
                                         compensate=compensate)
        parity.check(f"attend {name} smc={int(compensate)} bh={bh}", O[b, hh, :w.n_valid], want, w.dtype)
        assert np.all(O[b, hh, w.n_valid:] == 0)


@pytest.mark.parametrize("name", ["cfg1", "lowrank-bf16-d64-n3900pad-c128", "lowrank-bf16-d128-n2048-c128",
                                  "fp32-d128-n640-c64", "single-cluster-n100-c128"])
def test_dense_attention(helpers, name):
    w = CASES[name]()
    run = helpers.Run(w)
    O = run.dense()
    for b in range(w.B):
        for hh in range(w.H):
            Qf, Kf, Vf = (x[b, hh, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
            rows = np.arange(0, w.n_valid, max(1, w.n_valid // 300))
            want = orc.dense_attention(Qf, Kf, Vf, rows=rows)
            parity.check(f"dense {name} bh={b * w.H + hh}", O[b, hh, rows], want, w.dtype)
            assert np.all(O[b, hh, w.n_valid:] == 0)


@pytest.mark.parametrize("name", ["cfg1", "lowrank-bf16-d64-n3900pad-c128", "grid-bf16-d128-c128"])
def test_forward_end_to_end_matches_oracle_forward(helpers, name):
    w = CASES[name]()
    run = helpers.Run(w)
    O = run.forward()
    for bh in range(w.B * w.H):
        b, hh = divmod(bh, w.H)
        Qf, Kf, Vf = (x[b, hh, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
        fr = orc.forward_head(Qf, Kf, Vf, w.c, w.k, seed=0, bh=bh)
        parity.check(f"forward {name} bh={bh}", O[b, hh, :w.n_valid], fr.O, w.dtype)
        # error against dense attention, GPU and oracle side by side
        rows = np.arange(0, w.n_valid, max(1, w.n_valid // 200))
        dense = orc.dense_attention(Qf, Kf, Vf, rows=rows)
        e_gpu = np.abs(O[b, hh, rows] - dense).max()
        e_orc = np.abs(fr.O[rows] - dense).max()
        assert abs(e_gpu - e_orc) <= TOL[w.dtype] + 1e-12


# ---------------------------------------------------------------------------
# Full-size workloads, in the launch configuration the benchmark uses:
# clustering bit-exact on sampled heads, routing exact, attention on sampled
# query clusters.
# ---------------------------------------------------------------------------

FULL = {
    2: dict(heads=list(range(8)), clusters_per_head=24),
    3: dict(heads=[0, 23], clusters_per_head=12),
    4: dict(heads=[2], clusters_per_head=12),
}


@pytest.mark.parametrize("cfg", [2, 3, 4])
def test_full_size_config(helpers, cfg):
    w = wl.config_workload(cfg)
    run = helpers.Run(w)
    run.forward()
    got = {k: v for k, v in run.cluster().items()}
    kept_gpu, bits_gpu = run.route()
    O = run.forward()
    rng = np.random.default_rng(cfg)
    for bh in FULL[cfg]["heads"]:
        b, hh = divmod(bh, w.H)
        Qf, Kf, Vf = (x[b, hh, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
        h = orc.cluster_head(Qf, Kf, w.c, seed=0, bh=bh)
        np.testing.assert_array_equal(got["perm_q"][bh], h.perm_q)
        np.testing.assert_array_equal(got["perm_k"][bh], h.perm_k)
        kept = orc.topk_route(orc.centroid_scores(h.qbar, h.kbar), w.k)
        np.testing.assert_array_equal(kept_gpu[bh], kept)
        sample = np.sort(rng.choice(run.C, size=FULL[cfg]["clusters_per_head"], replace=False))
        sample = np.unique(np.append(sample, run.C - 1))   # include the ragged last cluster
        want = orc.compensated_attention(Qf, Kf, Vf, h.perm_q, h.count_q, h.perm_k, h.count_k, kept, w.c,
                                         clusters=sample)
        rows = np.concatenate([h.perm_q[a * w.c: a * w.c + h.count_q[a]] for a in sample])
        parity.check(f"full-size cfg{cfg} bh={bh} ({len(sample)} clusters)", O[b, hh, rows], want[rows], w.dtype)
