"""Upload workloads, call the C ABI, download results (GPU tests only)."""
from __future__ import annotations

import numpy as np

import free_clustered_block_b200 as ca


def torch():
    import torch as _t
    return _t


def check_device_error():
    """Every bounded wait in the kernels reports a timeout through the
    library's device error word; a GPU test must see it clear."""
    st = ca.ca_get_device_error()
    assert st == ca.CA_OK, f"device error: {ca.status_string(st)}"


def dev_tensor(x: np.ndarray, dtype: str):
    """float32 numpy (bf16-exact for bf16 workloads) -> contiguous CUDA tensor."""
    t = torch()
    h = t.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        h = h.to(t.bfloat16)
    return h.cuda().contiguous()


def shape_of(w, n_valid=None):
    return ca.make_shape(w.B, w.H, w.N_alloc, w.n_valid if n_valid is None else n_valid, w.d, w.c,
                         ca.CA_BF16 if w.dtype == "bf16" else ca.CA_FP32)


class Run:
    """Device buffers for one workload and the C-ABI calls on them."""

    def __init__(self, w, k=None, compensate=None, seed=0, power_iters=8, transform=True, selection="topk",
                 recall=0.9, min_count=16, clustering="split", c_k=0):
        t = torch()
        self.w = w
        self.k = w.k if k is None else k
        self.compensate = w.compensate if compensate is None else compensate
        self.Q = dev_tensor(w.Q, w.dtype)
        self.K = dev_tensor(w.K, w.dtype)
        self.V = dev_tensor(w.V, w.dtype)
        self.O = t.empty_like(self.Q)
        self.layer = ca.ClusterAttention(w.B, w.H, w.N_alloc, w.n_valid, w.d, w.c, self.k, dtype=w.dtype,
                                         compensate=self.compensate, power_iters=power_iters,
                                         transform=transform, seed=seed, selection=selection, recall=recall,
                                         min_count=min_count, clustering=clustering, c_k=c_k)
        self.C = self.layer.C
        self.Ck = self.layer.Ck
        self.ck = self.layer.c_k

    def cluster(self):
        self.layer.cluster(self.Q, self.K)
        t = torch(); t.cuda.synchronize()
        check_device_error()
        b = self.layer.buf
        BH, C, c, d = self.w.B * self.w.H, self.C, self.w.c, self.w.d
        Ck, ck = self.Ck, self.ck
        return dict(perm_q=b.perm_q.cpu().numpy().reshape(BH, C * c),
                    perm_k=b.perm_k.cpu().numpy().reshape(BH, Ck * ck),
                    count_q=b.count_q.cpu().numpy().reshape(BH, C),
                    count_k=b.count_k.cpu().numpy().reshape(BH, Ck),
                    qbar=b.qbar.cpu().numpy().reshape(BH, C, d),
                    kbar=b.kbar.cpu().numpy().reshape(BH, Ck, d))

    def set_clusters(self, heads):
        """Overwrite the device cluster buffers with oracle results (list over bh)."""
        t = torch()
        b = self.layer.buf
        b.perm_q.copy_(t.from_numpy(np.concatenate([h.perm_q for h in heads]).astype(np.int32)))
        b.perm_k.copy_(t.from_numpy(np.concatenate([h.perm_k for h in heads]).astype(np.int32)))
        b.count_q.copy_(t.from_numpy(np.concatenate([h.count_q for h in heads]).astype(np.int32)))
        b.count_k.copy_(t.from_numpy(np.concatenate([h.count_k for h in heads]).astype(np.int32)))
        b.qbar.copy_(t.from_numpy(np.concatenate([h.qbar.ravel() for h in heads])))
        b.kbar.copy_(t.from_numpy(np.concatenate([h.kbar.ravel() for h in heads])))

    def route(self):
        self.layer.route()
        t = torch(); t.cuda.synchronize()
        check_device_error()
        b = self.layer.buf
        BH, C = self.w.B * self.w.H, self.C
        W = (self.Ck + 31) // 32
        return (b.kept_idx.cpu().numpy().reshape(BH, C, self.k),
                b.kept_bits.cpu().numpy().view(np.uint32).reshape(BH, C, W))

    def route_counts(self):
        """Per-query-cluster kept counts [BH, C] (adaptive selection)."""
        b = self.layer.buf
        return b.kept_count.cpu().numpy().reshape(self.w.B * self.w.H, self.C)

    def set_routes(self, kept_list):
        from oracle import ca_oracle as orc
        t = torch()
        b = self.layer.buf
        b.kept_idx.copy_(t.from_numpy(np.concatenate([k.ravel() for k in kept_list]).astype(np.int32)))
        bits = np.concatenate([orc.route_bits(k, self.Ck).ravel() for k in kept_list])
        b.kept_bits.copy_(t.from_numpy(bits.view(np.int32)))

    def attend(self):
        self.layer.attend(self.Q, self.K, self.V, self.O)
        t = torch(); t.cuda.synchronize()
        check_device_error()
        return self.O.float().cpu().numpy()

    def dense(self):
        t = torch()
        O = t.empty_like(self.Q)
        self.layer.dense(self.Q, self.K, self.V, O)
        t.cuda.synchronize()
        check_device_error()
        return O.float().cpu().numpy()

    def forward(self):
        self.layer(self.Q, self.K, self.V, self.O)
        t = torch(); t.cuda.synchronize()
        check_device_error()
        return self.O.float().cpu().numpy()
