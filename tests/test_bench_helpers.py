"""The benchmark's work definitions, on CPU: algorithmic FLOPs of the
attention step and of dense attention, clustering levels and row bytes, for
the three full-size configurations, against the figures computed from the
shapes alone (kept blocks 4 n (k c) d H, compensation 4 n (C - k) d H over
the excluded clusters, dense 4 n^2 d H, rows read once per level by both
tensors)."""
from types import SimpleNamespace

import pytest

import bench
import free_clustered_block_b200 as ca

CFG = {
    # B, H, N_alloc, n_valid, d, c, k, levels of the split tree
    2: (1, 8, 65536, 65536, 64, 128, 64, 9),
    3: (1, 40, 76800, 75600, 128, 128, 89, 10),
    4: (1, 4, 262144, 262144, 64, 256, 64, 10),
}


def _w(cfg):
    B, H, N, n, d, c, k, _ = CFG[cfg]
    return SimpleNamespace(B=B, H=H, N_alloc=N, n_valid=n, d=d, c=c, k=k, C=-(-n // c), dtype="bf16",
                           compensate=True, name=f"cfg{cfg}")


@pytest.mark.parametrize("cfg,kept_tf,dense_tf", [(2, 1.100, 8.80), (3, 17.64, 117.0), (4, 4.40, 70.4)])
def test_attention_and_dense_flops(cfg, kept_tf, dense_tf):
    w = _w(cfg)
    kept, smc = bench.attention_flops(w)
    assert kept == 4.0 * w.n_valid * w.k * w.c * w.d * w.H
    assert smc == 4.0 * w.n_valid * (w.C - w.k) * w.d * w.H
    assert kept / 1e12 == pytest.approx(kept_tf, abs=0.01)
    assert bench.dense_flops(w) / 1e12 == pytest.approx(dense_tf, rel=2e-3)
    w.compensate = False
    assert bench.attention_flops(w)[1] == 0.0


def test_unequal_key_cluster_size_changes_the_key_side_only():
    w = _w(2)
    w.c, w.c_k = 64, 128
    kept, smc = bench.attention_flops(w)
    assert kept == 4.0 * w.n_valid * w.k * 128 * w.d * w.H
    assert smc == 4.0 * w.n_valid * (512 - w.k) * w.d * w.H


@pytest.mark.parametrize("cfg,gb", [(2, 1.21), (3, 15.5), (4, 2.68)])
def test_cluster_levels_and_row_bytes(cfg, gb):
    B, H, N, n, d, c, k, levels = CFG[cfg]
    shape = ca.make_shape(B, H, N, n, d, c, ca.CA_BF16)
    assert bench.cluster_levels(ca, shape) == levels
    assert bench.cluster_row_bytes(_w(cfg), levels) / 1e9 == pytest.approx(gb, abs=0.03)   # figures rounded


def test_capture_table_is_keyed_by_workload():
    assert bench.attention_capture("no-such-workload") is None
    for c in bench.ATTN_CAPTURES:
        assert set(c) >= {"sha", "workload", "traffic", "tensor_pipe_pct"}
        assert c["traffic"] > 0 and 0 < c["tensor_pipe_pct"] < 100
