"""Token-major input (CA_LAYOUT_BNHD, [B, N, H_total, d]) on the GPU.

The layout changes only where the kernels read Q, K, V and write O, never
the arithmetic: the partitions, routes and outputs must equal the head-major
call's bit for bit. A slice of heads of a token-major tensor (pointers offset
to the first head, H_total > H, head_base) must equal those heads of the
whole call, and leave the other heads' output untouched; the oracle check at
the end ties one token-major forward to the fp64 oracle directly.
"""
import numpy as np
import pytest

import workloads as wl
from oracle import ca_oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu

CASES = {
    "bf16-d64-n3900pad-c128": lambda: wl.make_workload("lowrank", B=2, H=3, N=4096, n_valid=3900, d=64, c=128,
                                                       k=6, dtype="bf16", seed=91),
    "bf16-d128-c128": lambda: wl.make_workload("grid", H=2, N=2048, d=128, c=128, k=4, dtype="bf16", seed=92,
                                               grid=(8, 16, 16)),
    "bf16-d64-c256": lambda: wl.make_workload("heavytail", H=2, N=4096, n_valid=4000, d=64, c=256, k=3,
                                              dtype="bf16", seed=93),
    "fp32-d64-n1000-c64": lambda: wl.make_workload("mixture", H=3, N=1024, n_valid=1000, d=64, c=64, k=5,
                                                   dtype="fp32", seed=94),
}


def _torch():
    import torch
    return torch


def _dev(x, dtype, layout):
    """[B, H, N, d] numpy -> CUDA tensor in the given layout."""
    torch = _torch()
    a = x if layout == "bhnd" else x.transpose(0, 2, 1, 3)
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.cuda().contiguous()


def _to_bhnd(O, layout):
    o = O.float().cpu().numpy()
    return o if layout == "bhnd" else o.transpose(0, 2, 1, 3)


def _forward(w, layout, c_k=0, dense=False):
    import free_clustered_block_b200 as ca
    torch = _torch()
    Q, K, V = (_dev(x, w.dtype, layout) for x in (w.Q, w.K, w.V))
    O = torch.full_like(Q, 5.0)
    layer = ca.ClusterAttention(w.B, w.H, w.N_alloc, w.n_valid, w.d, w.c, w.k, dtype=w.dtype, layout=layout,
                                c_k=c_k)
    if dense:
        layer.dense(Q, K, V, O)
    else:
        layer(Q, K, V, O)
    torch.cuda.synchronize()
    assert ca.ca_get_device_error() == ca.CA_OK
    perms = None if dense else (layer.buf.perm_q.cpu().numpy(), layer.buf.perm_k.cpu().numpy())
    return _to_bhnd(O, layout), perms


@pytest.mark.parametrize("name", list(CASES))
def test_token_major_forward_equals_head_major(name):
    w = CASES[name]()
    O1, p1 = _forward(w, "bhnd")
    O2, p2 = _forward(w, "bnhd")
    np.testing.assert_array_equal(p1[0], p2[0])
    np.testing.assert_array_equal(p1[1], p2[1])
    np.testing.assert_array_equal(O1, O2)
    assert np.all(O2[:, :, w.n_valid:] == 0)


@pytest.mark.parametrize("name", ["bf16-d64-n3900pad-c128", "bf16-d128-c128", "fp32-d64-n1000-c64"])
def test_token_major_dense_equals_head_major(name):
    w = CASES[name]()
    O1, _ = _forward(w, "bhnd", dense=True)
    O2, _ = _forward(w, "bnhd", dense=True)
    np.testing.assert_array_equal(O1, O2)
    assert np.all(O2[:, :, w.n_valid:] == 0)


def test_token_major_unequal_cluster_sizes():
    w = wl.make_workload("lowrank", H=2, N=4096, n_valid=4000, d=64, c=64, k=8, dtype="bf16", seed=95)
    O1, p1 = _forward(w, "bhnd", c_k=128)
    O2, p2 = _forward(w, "bnhd", c_k=128)
    np.testing.assert_array_equal(p1[1], p2[1])
    np.testing.assert_array_equal(O1, O2)


def test_token_major_head_slice():
    # heads 1..2 of a 4-head token-major tensor: pointers offset by one head,
    # H = 2, H_total = 4, head_base = 1
    import free_clustered_block_b200 as ca
    torch = _torch()
    w = wl.make_workload("lowrank", H=4, N=2048, n_valid=2000, d=64, c=128, k=4, dtype="bf16", seed=96)
    Q, K, V = (_dev(x, "bf16", "bnhd") for x in (w.Q, w.K, w.V))
    O_full = torch.full_like(Q, 5.0)
    full = ca.ClusterAttention(w.B, w.H, w.N_alloc, w.n_valid, w.d, w.c, w.k, layout="bnhd")
    full(Q, K, V, O_full)
    O_part = torch.full_like(Q, 5.0)
    part = ca.ClusterAttention(w.B, 2, w.N_alloc, w.n_valid, w.d, w.c, w.k, layout="bnhd", H_total=4, head_base=1)
    sl = lambda t: t[:, :, 1:3, :]   # a view: data pointer offset by one head, token stride 4 d
    part(sl(Q), sl(K), sl(V), sl(O_part))
    torch.cuda.synchronize()
    assert ca.ca_get_device_error() == ca.CA_OK
    assert torch.equal(O_part[:, :, 1:3], O_full[:, :, 1:3])
    assert torch.all(O_part[:, :, 0] == 5.0) and torch.all(O_part[:, :, 3] == 5.0)


def test_token_major_host_forward():
    import free_clustered_block_b200 as ca
    torch = _torch()
    w = wl.make_workload("lowrank", B=2, H=3, N=2048, n_valid=1900, d=64, c=128, k=3, dtype="bf16", seed=97)
    Q, K, V = (_dev(x, "bf16", "bnhd") for x in (w.Q, w.K, w.V))
    layer = ca.ClusterAttention(w.B, w.H, w.N_alloc, w.n_valid, w.d, w.c, w.k, layout="bnhd")
    Od = torch.empty_like(Q)
    layer.forward_fused(Q, K, V, Od)
    torch.cuda.synchronize()
    hQ, hK, hV = (x.cpu().pin_memory() for x in (Q, K, V))
    hO = torch.full_like(hQ, 7.0).pin_memory()
    ws = torch.empty(ca.forward_host_workspace_bytes(layer.shape, w.k), dtype=torch.uint8, device="cuda")
    ca.ca_forward_host(hQ, hK, hV, layer.shape, layer.params, w.k, True, hO, ws)
    assert ca.ca_get_device_error() == ca.CA_OK
    assert torch.equal(Od.cpu(), hO)


def test_token_major_against_the_oracle():
    w = CASES["bf16-d64-n3900pad-c128"]()
    O, _ = _forward(w, "bnhd")
    for bh in range(w.B * w.H):
        b, h = divmod(bh, w.H)
        Qf, Kf, Vf = (x[b, h, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
        fr = orc.forward_head(Qf, Kf, Vf, w.c, w.k, seed=0, bh=bh)
        parity.check(f"token-major forward bh={bh}", O[b, h, :w.n_valid], fr.O, w.dtype)
