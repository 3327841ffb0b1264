"""Failure detection without a GPU fault. Every device-side wait of the
tensor-core kernels is bounded by %globaltimer (ca_set_wait_limit): a wait that
runs out sets CA_ERR_TIMEOUT in the device error word and the kernel returns.
ca_check_bounded_wait runs that same wait on an mbarrier that nothing
completes, so it must run out; the context stays usable afterwards and the
attention that follows is correct."""
import time

import numpy as np
import pytest

import free_clustered_block_b200 as ca
import workloads as wl
from oracle import ca_oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


def test_completed_wait_reports_ok():
    import torch
    torch.cuda.init()
    assert ca.ca_get_device_error() == ca.CA_OK
    assert ca.ca_check_bounded_wait(1_000_000, True) == ca.CA_OK
    assert ca.ca_get_device_error() == ca.CA_OK


def test_wait_nothing_completes_times_out_and_the_context_recovers():
    from tests import gpu_helpers as gh
    import torch
    torch.cuda.init()
    assert ca.ca_get_device_error() == ca.CA_OK
    t0 = time.perf_counter()
    assert ca.ca_check_bounded_wait(2_000_000, False) == ca.CA_OK   # 2 ms limit
    st = ca.ca_get_device_error()          # synchronises, reads and clears the word
    elapsed = time.perf_counter() - t0
    assert st == ca.CA_ERR_TIMEOUT, ca.status_string(st)
    assert elapsed < 5.0                   # the kernel returned; nothing hung
    assert ca.ca_get_device_error() == ca.CA_OK   # the word was cleared
    assert ca.ca_check_bounded_wait(0, False) == ca.CA_ERR_INVALID_ARG

    # the same context: attention with the default limit is correct
    w = wl.make_workload("lowrank", H=2, N=2048, d=64, c=128, k=4, dtype="bf16", seed=51)
    run = gh.Run(w)
    ref = orc.cluster_workload(w.Q.astype(np.float64), w.K.astype(np.float64), w.n_valid, w.c, seed=0)
    kept = [orc.topk_route(orc.centroid_scores(h.qbar, h.kbar), run.k) for h in ref]
    run.set_clusters(ref)
    run.set_routes(kept)
    O = run.attend()
    assert ca.ca_get_device_error() == ca.CA_OK
    for bh, h in enumerate(ref):
        b, hh = divmod(bh, w.H)
        Qf, Kf, Vf = (x[b, hh, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
        want = orc.compensated_attention(Qf, Kf, Vf, h.perm_q, h.count_q, h.perm_k, h.count_k, kept[bh], w.c)
        parity.check(f"after a timeout bh={bh}", O[b, hh, :w.n_valid], want, w.dtype)
