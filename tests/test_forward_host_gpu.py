"""ca_forward_host: host buffers in and out, the heads pipelined in groups
(the copies of one group overlapping the forward of another). Its output must
equal ca_forward on device buffers bit for bit: the groups are keyed by their
global head index, so the clusters and the attention are the same."""
import numpy as np
import pytest

import workloads as wl

pytestmark = pytest.mark.gpu


def _both(w, head_base=0, pinned=True):
    import torch
    import free_clustered_block_b200 as ca
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).cuda()
    Q, K, V = dev(w.Q), dev(w.K), dev(w.V)
    layer = ca.ClusterAttention(w.B, w.H, w.N_alloc, w.n_valid, w.d, w.c, w.k, dtype="bf16", head_base=head_base)
    Od = torch.empty_like(Q)
    layer.forward_fused(Q, K, V, Od)
    torch.cuda.synchronize()
    hQ, hK, hV = (x.cpu() for x in (Q, K, V))
    hO = torch.full_like(hQ, 7.0)
    if pinned:
        hQ, hK, hV, hO = (x.pin_memory() for x in (hQ, hK, hV, hO))
    ws = torch.empty(ca.forward_host_workspace_bytes(layer.shape, w.k), dtype=torch.uint8, device="cuda")
    ca.ca_forward_host(hQ, hK, hV, layer.shape, layer.params, w.k, True, hO, ws)
    assert ca.ca_get_device_error() == ca.CA_OK
    return Od.cpu(), hO


@pytest.mark.parametrize("B,H", [(1, 5), (1, 2), (2, 3), (1, 1)])
def test_pipelined_host_forward_equals_device_forward(B, H):
    import torch
    w = wl.make_workload("lowrank", B=B, H=H, N=2048, n_valid=2000, d=64, c=128, k=3, dtype="bf16", seed=81)
    Od, Oh = _both(w)
    assert torch.equal(Od, Oh)
    assert torch.all(Oh[:, :, w.n_valid:] == 0)


def test_pipelined_host_forward_with_head_base_and_pageable_memory():
    import torch
    w = wl.make_workload("grid", H=3, N=1536, d=128, c=128, k=2, dtype="bf16", seed=82, grid=(8, 12, 16))
    Od, Oh = _both(w, head_base=5, pinned=False)
    assert torch.equal(Od, Oh)
