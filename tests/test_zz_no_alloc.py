"""ca_cluster_noalloc: clustering with the library's fixed device scratch,
for callers that cannot allocate device memory (plugins inside frameworks
that own every allocation, loops that must not call cudaMalloc).

Checked through the C ABI against ca_cluster (the entry point that takes a
caller workspace) on two calls in a row with different inputs, so the second
call also shows that the first call's leftovers in the shared scratch do not
leak into its result. Runs last (file name) so a failure here leaves every
other test already run; it passes alone and after the others.
"""
import ctypes

import numpy as np
import pytest

import workloads as wl

pytestmark = pytest.mark.gpu


def _run_both(helpers, w):
    import torch
    import free_clustered_block_b200 as ca
    run = helpers.Run(w)
    ref = run.cluster()                                    # ca_cluster with a workspace
    BH, C, c, d = w.B * w.H, run.C, w.c, w.d
    i32, f64 = torch.int32, torch.float64
    bufs = dict(perm_q=torch.full((BH * C * c,), 7, dtype=i32, device="cuda"),
                perm_k=torch.full((BH * C * c,), 7, dtype=i32, device="cuda"),
                count_q=torch.zeros(BH * C, dtype=i32, device="cuda"),
                count_k=torch.zeros(BH * C, dtype=i32, device="cuda"),
                qbar=torch.zeros(BH * C * d, dtype=f64, device="cuda"),
                kbar=torch.zeros(BH * C * d, dtype=f64, device="cuda"))
    cl = ca.clusters_struct(bufs["perm_q"], bufs["perm_k"], bufs["count_q"], bufs["count_k"], bufs["qbar"],
                            bufs["kbar"])
    st = ca.lib().ca_cluster_noalloc(ctypes.c_void_p(run.Q.data_ptr()), ctypes.c_void_p(run.K.data_ptr()),
                                     ctypes.byref(run.layer.shape), ctypes.byref(run.layer.params),
                                     ctypes.byref(cl), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == ca.CA_OK, ca.status_string(st)
    torch.cuda.synchronize()
    assert ca.ca_get_device_error() == ca.CA_OK
    got = {k: v.cpu().numpy() for k, v in bufs.items()}
    for key in ("perm_q", "perm_k", "count_q", "count_k"):
        np.testing.assert_array_equal(got[key].reshape(ref[key].shape), ref[key])
    for key in ("qbar", "kbar"):
        r = ref[key]
        assert np.abs(got[key].reshape(r.shape) - r).max() <= 1e-12 * max(1.0, np.abs(r).max())


def test_noalloc_cluster_matches_workspace_cluster_twice():
    from tests import gpu_helpers
    a = wl.make_workload("lowrank", H=2, N=4096, n_valid=4000, d=64, c=128, k=4, dtype="bf16", seed=31)
    b = wl.make_workload("mixture", H=2, N=4096, n_valid=4000, d=64, c=128, k=4, dtype="bf16", seed=32)
    _run_both(gpu_helpers, a)
    _run_both(gpu_helpers, b)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import free_clustered_block_b200 as ca
    big = ca.make_shape(1, 8, 65536, 65536, 64, 128, ca.CA_BF16)     # needs ~45 MiB
    assert ca.cluster_workspace_bytes(big) > (16 << 20)
    cl = ca.ca_clusters(0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000)
    st = ca.lib().ca_cluster_noalloc(ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), ctypes.byref(big),
                                     None, ctypes.byref(cl), None)
    assert st == ca.CA_ERR_WORKSPACE
