"""Diagonalized recursive splitting on the GPU vs the fp64 oracle
("ClusterAttention", Section 3.2.1 "Diagonalized recursive splitting"):
the principal-component basis from the GPU's Jacobi eigensolver, the
per-set highest-variance coordinate and the split. Bar: partitions
bit-exact, centroids to 1e-12, the whole layer's attention as in the main
parity tests."""
import numpy as np
import pytest

import workloads as wl
from oracle import ca_oracle as orc

from tests import parity

pytestmark = pytest.mark.gpu

CASES = {
    "lowrank-bf16-d64-n3900pad-c128": lambda: wl.make_workload("lowrank", H=2, N=4096, n_valid=3900, d=64, c=128,
                                                               k=6, dtype="bf16", seed=41),
    "mix-fp32-d64-n1000-c64": lambda: wl.make_workload("mixture", H=2, N=1000, d=64, c=64, k=5, dtype="fp32",
                                                       seed=42),
    "grid-bf16-d128-c128": lambda: wl.make_workload("grid", H=1, N=6144, d=128, c=128, k=7, dtype="bf16", seed=43,
                                                    grid=(8, 9, 80)),
    "heavytail-bf16-d64-c64": lambda: wl.make_workload("heavytail", H=2, N=5000, d=64, c=64, k=9, dtype="bf16",
                                                       seed=44),
    "mix-fp32-d128-n2c+1": lambda: wl.make_workload("mixture", H=1, N=257, d=128, c=128, k=2, dtype="fp32",
                                                    seed=45),
}


def _heads(w):
    return [(b, h, w.Q[b, h, :w.n_valid].astype(np.float64), w.K[b, h, :w.n_valid].astype(np.float64))
            for b in range(w.B) for h in range(w.H)]


def _check_partition(got, bh, ref):
    np.testing.assert_array_equal(got["perm_q"][bh], ref.perm_q)
    np.testing.assert_array_equal(got["perm_k"][bh], ref.perm_k)
    np.testing.assert_array_equal(got["count_q"][bh], ref.count_q)
    np.testing.assert_array_equal(got["count_k"][bh], ref.count_k)
    assert np.abs(got["qbar"][bh] - ref.qbar).max() <= 1e-12 * max(1.0, np.abs(ref.qbar).max())
    assert np.abs(got["kbar"][bh] - ref.kbar).max() <= 1e-12 * max(1.0, np.abs(ref.kbar).max())


@pytest.mark.parametrize("form", ["topk", "adaptive", "untransformed"])
@pytest.mark.parametrize("name", list(CASES))
def test_diagonal_partition_bit_exact(name, form):
    from tests import gpu_helpers as gh
    w = CASES[name]()
    transform = form != "untransformed"
    run = gh.Run(w, clustering="diagonal", seed=7, transform=transform,
                 selection="adaptive" if form == "adaptive" else "topk")
    got = run.cluster()
    for bh, (b, h, Qf, Kf) in enumerate(_heads(w)):
        ref = orc.cluster_head(Qf, Kf, w.c, seed=7, bh=bh, transform=transform,
                               query_form="adaptive" if form == "adaptive" else "topk", splitting="diagonal")
        _check_partition(got, bh, ref)


def test_diagonal_partition_full_size_heads():
    # B=1 H=8 N=65,536 d=64 c=128: all heads clustered on the GPU, two checked
    from tests import gpu_helpers as gh
    w = wl.make_workload("lowrank", H=8, N=65536, d=64, c=128, k=64, dtype="bf16", seed=2)
    run = gh.Run(w, clustering="diagonal")
    got = run.cluster()
    for bh in (0, 7):
        Qf = w.Q[0, bh, :w.n_valid].astype(np.float64)
        Kf = w.K[0, bh, :w.n_valid].astype(np.float64)
        ref = orc.cluster_head(Qf, Kf, w.c, seed=0, bh=bh, splitting="diagonal")
        _check_partition(got, bh, ref)


@pytest.mark.parametrize("name", ["lowrank-bf16-d64-n3900pad-c128", "mix-fp32-d64-n1000-c64",
                                  "grid-bf16-d128-c128"])
def test_diagonal_end_to_end(name):
    from tests import gpu_helpers as gh
    w = CASES[name]()
    run = gh.Run(w, clustering="diagonal", seed=7)
    O = run.forward()
    for bh, (b, h, Qf, Kf) in enumerate(_heads(w)):
        Vf = w.V[b, h, :w.n_valid].astype(np.float64)
        ref = orc.cluster_head(Qf, Kf, w.c, seed=7, bh=bh, splitting="diagonal")
        kept = orc.topk_route(orc.centroid_scores(ref.qbar, ref.kbar), w.k)
        want = orc.compensated_attention(Qf, Kf, Vf, ref.perm_q, ref.count_q, ref.perm_k, ref.count_k, kept, w.c,
                                         compensate=w.compensate)
        parity.check(f"diagonal {name} bh={bh}", O[b, h, :w.n_valid], want, w.dtype)
