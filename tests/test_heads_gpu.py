"""One layer split by heads: a call on a slice of the heads (pointers offset
to the slice, H = the slice's length, ca_cluster_params.head_base = the
slice's first flattened head index) must give exactly what the whole-layer
call gives for those heads, and what the oracle gives for their global
indices. This is each GPU's share when a layer is divided across GPUs."""
import numpy as np
import pytest

import workloads as wl
from oracle import ca_oracle as orc

pytestmark = pytest.mark.gpu


def _run(layer_args, Q, K, V, head_base):
    import torch
    import free_clustered_block_b200 as ca
    B, H, N, nv, d, c, k = layer_args
    layer = ca.ClusterAttention(B, H, N, nv, d, c, k, dtype="bf16", head_base=head_base)
    O = layer(Q, K, V)
    torch.cuda.synchronize()
    assert ca.ca_get_device_error() == ca.CA_OK
    C = layer.C
    return (layer.buf.perm_q.cpu().numpy().reshape(B * H, C * c), layer.buf.perm_k.cpu().numpy().reshape(B * H, C * c),
            O.float().cpu().numpy().reshape(B * H, N, d))


@pytest.mark.parametrize("B,H,lo,hi", [(1, 4, 1, 3), (2, 2, 1, 3), (1, 4, 3, 4)])
def test_head_slice_reproduces_the_whole_layer(B, H, lo, hi):
    import torch
    w = wl.make_workload("lowrank", B=B, H=H, N=4096, n_valid=4000, d=64, c=128, k=4, dtype="bf16", seed=71)

    def dev(x):
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).cuda().contiguous()

    Q, K, V = dev(w.Q), dev(w.K), dev(w.V)
    full_pq, full_pk, full_O = _run((B, H, w.N_alloc, w.n_valid, w.d, w.c, w.k), Q, K, V, 0)
    # the slice of flattened heads [lo, hi): contiguous memory, presented as B = 1, H = hi - lo
    fl = lambda t: t.reshape(B * H, w.N_alloc, w.d)[lo:hi].reshape(1, hi - lo, w.N_alloc, w.d)
    Qs, Ks, Vs = fl(Q), fl(K), fl(V)
    assert Qs.data_ptr() == Q.data_ptr() + lo * w.N_alloc * w.d * 2     # a view, no copy
    pq, pk, O = _run((1, hi - lo, w.N_alloc, w.n_valid, w.d, w.c, w.k), Qs, Ks, Vs, lo)
    np.testing.assert_array_equal(pq, full_pq[lo:hi])
    np.testing.assert_array_equal(pk, full_pk[lo:hi])
    np.testing.assert_array_equal(O, full_O[lo:hi])                     # same arithmetic, bit for bit
    for i, bh in enumerate(range(lo, hi)):
        b, h = divmod(bh, H)
        Qf, Kf = (x[b, h, :w.n_valid].astype(np.float64) for x in (w.Q, w.K))
        ref = orc.cluster_head(Qf, Kf, w.c, seed=0, bh=bh)
        np.testing.assert_array_equal(pq[i], ref.perm_q)
        np.testing.assert_array_equal(pk[i], ref.perm_k)


def test_slice_without_head_base_differs():
    """The offset matters: the same slice keyed as heads 0.. draws other samples."""
    import torch
    w = wl.make_workload("lowrank", H=4, N=4096, n_valid=4000, d=64, c=128, k=4, dtype="bf16", seed=72)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).cuda()
    Q, K, V = dev(w.Q), dev(w.K), dev(w.V)
    pq1, _, _ = _run((1, 2, w.N_alloc, w.n_valid, w.d, w.c, w.k), Q[:, 2:4].contiguous(), K[:, 2:4].contiguous(),
                     V[:, 2:4].contiguous(), 2)
    pq0, _, _ = _run((1, 2, w.N_alloc, w.n_valid, w.d, w.c, w.k), Q[:, 2:4].contiguous(), K[:, 2:4].contiguous(),
                     V[:, 2:4].contiguous(), 0)
    assert not np.array_equal(pq1, pq0)
