"""Ablations on the GPU vs the fp64 oracle: the random-cluster baseline of the
paper's error analysis ("ClusterAttention", Section 1.2 and Section 4) and the
untransformed split (transform off, Section 3.2.2). Bar: partitions
bit-exact, centroids to 1e-12, attention as in the main parity tests."""
import numpy as np
import pytest

import workloads as wl
from oracle import ca_oracle as orc

from tests import parity

pytestmark = pytest.mark.gpu

CASES = {
    "lowrank-bf16-d64-n3900pad-c128": lambda: wl.make_workload("lowrank", H=2, N=4096, n_valid=3900, d=64, c=128,
                                                               k=6, dtype="bf16", seed=31),
    "mix-fp32-d64-n1000-c64": lambda: wl.make_workload("mixture", H=2, N=1000, d=64, c=64, k=5, dtype="fp32",
                                                       seed=32),
    "grid-bf16-d128-c128": lambda: wl.make_workload("grid", H=1, N=6144, d=128, c=128, k=7, dtype="bf16", seed=33,
                                                    grid=(8, 9, 80)),
}


def _heads(w):
    return [(b, h, w.Q[b, h, :w.n_valid].astype(np.float64), w.K[b, h, :w.n_valid].astype(np.float64))
            for b in range(w.B) for h in range(w.H)]


@pytest.mark.parametrize("name", list(CASES))
def test_random_clusters_bit_exact(name):
    from tests import gpu_helpers as gh
    w = CASES[name]()
    run = gh.Run(w, clustering="random", seed=5)
    got = run.cluster()
    for bh, (b, h, Qf, Kf) in enumerate(_heads(w)):
        ref = orc.cluster_head_random(Qf, Kf, w.c, seed=5, bh=bh)
        np.testing.assert_array_equal(got["perm_q"][bh], ref.perm_q)
        np.testing.assert_array_equal(got["perm_k"][bh], ref.perm_k)
        np.testing.assert_array_equal(got["count_q"][bh], ref.count_q)
        assert np.abs(got["qbar"][bh] - ref.qbar).max() <= 1e-12 * max(1.0, np.abs(ref.qbar).max())
        assert np.abs(got["kbar"][bh] - ref.kbar).max() <= 1e-12 * max(1.0, np.abs(ref.kbar).max())


@pytest.mark.parametrize("compensate", [True, False])
@pytest.mark.parametrize("name", list(CASES))
def test_random_clusters_end_to_end(name, compensate):
    # the whole layer (random clusters, routing, attention) against the oracle
    from tests import gpu_helpers as gh
    w = CASES[name]()
    run = gh.Run(w, clustering="random", seed=5, compensate=compensate)
    O = run.forward()
    for bh, (b, h, Qf, Kf) in enumerate(_heads(w)):
        Vf = w.V[b, h, :w.n_valid].astype(np.float64)
        ref = orc.cluster_head_random(Qf, Kf, w.c, seed=5, bh=bh)
        kept = orc.topk_route(orc.centroid_scores(ref.qbar, ref.kbar), w.k)
        want = orc.compensated_attention(Qf, Kf, Vf, ref.perm_q, ref.count_q, ref.perm_k, ref.count_k, kept, w.c,
                                         compensate=compensate)
        parity.check(f"random clusters {name} smc={int(compensate)} bh={bh}", O[b, h, :w.n_valid], want, w.dtype)


@pytest.mark.parametrize("name", list(CASES))
def test_untransformed_split_bit_exact(name):
    from tests import gpu_helpers as gh
    w = CASES[name]()
    run = gh.Run(w, transform=False)
    got = run.cluster()
    for bh, (b, h, Qf, Kf) in enumerate(_heads(w)):
        ref = orc.cluster_head(Qf, Kf, w.c, seed=0, bh=bh, transform=False)
        np.testing.assert_array_equal(got["perm_q"][bh], ref.perm_q, err_msg=f"margin {ref.min_margin_q:.3g}")
        np.testing.assert_array_equal(got["perm_k"][bh], ref.perm_k, err_msg=f"margin {ref.min_margin_k:.3g}")
