"""Convenience holder of the buffers one ClusterAttention layer needs.

Allocates (with torch) the cluster, route and workspace buffers for one
shape and calls the C ABI; no computation happens here.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

from . import (CA_BF16, CA_FP32, CA_LAYOUT_BHND, CA_LAYOUT_BNHD, ca_attend, ca_attend_prepare, ca_attend_prepared, ca_cluster, num_key_clusters, ca_dense_attend, ca_forward, ca_route, ca_route_adaptive,
               attend_workspace_bytes, cluster_workspace_bytes, clusters_struct, forward_workspace_bytes,
               make_params, make_shape, num_clusters, routes_struct)


CLUSTERING_METHODS = {"split": 0, "random": 1, "diagonal": 2}


@dataclass
class Buffers:
    perm_q: object
    perm_k: object
    count_q: object
    count_k: object
    qbar: object
    kbar: object
    kept_idx: object
    kept_bits: object
    kept_count: object


class ClusterAttention:
    """One layer's shape, knobs and device buffers.

    clustering: "split" (basic recursive splitting, power iteration per set),
    "diagonal" (diagonalized recursive splitting) or "random" (random
    clusters, the error-analysis baseline).

    Q, K, V, O: torch CUDA tensors [B, H, N_alloc, d], bf16 or fp32, contiguous.

    c_k: key cluster size (0: the same as c, the query cluster size); the
    paper's evaluated blocks are c = 64 queries against c_k = 128 keys.

    head_base: global index of the first (b, h) pair these tensors hold, when
    they are a slice of a larger layer's heads (one GPU's share of a layer
    split across GPUs); the clusters are then those the whole layer would get.
    """

    def __init__(self, B: int, H: int, N_alloc: int, n_valid: int, d: int, c: int, k: int,
                 dtype: str = "bf16", compensate: bool = True, power_iters: int = 8,
                 sample_factor: int = 1, transform: bool = True, seed: int = 0, device="cuda",
                 selection: str = "topk", recall: float = 0.9, min_count: int = 16,
                 clustering: str = "split", head_base: int = 0, c_k: int = 0, layout: str = "bhnd",
                 H_total: int = 0):
        import torch
        self.torch = torch
        self.dtype_code = CA_BF16 if dtype == "bf16" else CA_FP32
        if layout not in ("bhnd", "bnhd"):
            raise ValueError("layout is 'bhnd' ([B, H, N, d]) or 'bnhd' ([B, N, H_total, d])")
        self.layout = layout
        self.shape = make_shape(B, H, N_alloc, n_valid, d, c, self.dtype_code, c_k,
                                CA_LAYOUT_BNHD if layout == "bnhd" else CA_LAYOUT_BHND, H_total)
        # adaptive selection pairs with the eq. 15 query representation
        self.selection = selection
        self.recall, self.min_count = recall, min_count
        self.params = make_params(power_iters, sample_factor, int(transform), seed,
                                  query_form=1 if selection == "adaptive" else 0,
                                  method=CLUSTERING_METHODS[clustering], head_base=head_base)
        self.k = k
        self.compensate = compensate
        C = num_clusters(self.shape)
        if C < 0:
            raise ValueError("invalid shape")
        Ck = num_key_clusters(self.shape)
        self.C, self.Ck = C, Ck
        self.c_k = c_k or c
        BH = B * H
        i32, f64 = torch.int32, torch.float64
        W = (Ck + 31) // 32
        self.buf = Buffers(
            perm_q=torch.empty(BH * C * c, dtype=i32, device=device),
            perm_k=torch.empty(BH * Ck * self.c_k, dtype=i32, device=device),
            count_q=torch.empty(BH * C, dtype=i32, device=device),
            count_k=torch.empty(BH * Ck, dtype=i32, device=device),
            qbar=torch.empty(BH * C * d, dtype=f64, device=device),
            kbar=torch.empty(BH * Ck * d, dtype=f64, device=device),
            kept_idx=torch.empty(BH * C * k, dtype=i32, device=device),
            kept_bits=torch.empty(BH * C * W, dtype=torch.int32, device=device),
            kept_count=torch.empty(BH * C, dtype=i32, device=device),
        )
        nbytes = max(cluster_workspace_bytes(self.shape), attend_workspace_bytes(self.shape))
        self.workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        self.fwd_workspace = None

    def clusters(self):
        b = self.buf
        return clusters_struct(b.perm_q, b.perm_k, b.count_q, b.count_k, b.qbar, b.kbar)

    def routes(self):
        # top-k rows hold exactly k; adaptive rows hold their own count (capacity k)
        count = self.buf.kept_count if self.selection == "adaptive" else None
        return routes_struct(self.k, self.buf.kept_idx, self.buf.kept_bits, count)

    def cluster(self, Q, K, stream=None):
        ca_cluster(Q, K, self.shape, self.params, self.clusters(), self.workspace, stream)

    def route(self, stream=None):
        if self.selection == "adaptive":
            ca_route_adaptive(self.shape, self.clusters(), self.recall, self.min_count, self.routes(), stream)
        else:
            ca_route(self.shape, self.clusters(), self.routes(), stream)

    def attend(self, Q, K, V, O, stream=None):
        ca_attend(Q, K, V, self.shape, self.clusters(), self.routes(), self.compensate, O, self.workspace,
                  stream)

    def attend_prepare(self, Q, K, V, stream=None):
        """ca_attend's first half (value centroids, cluster-ordered copies)."""
        ca_attend_prepare(Q, K, V, self.shape, self.clusters(), self.workspace, stream)

    def attend_prepared(self, Q, K, V, O, stream=None):
        """ca_attend's second half: the attention kernel on the prepared workspace."""
        ca_attend_prepared(Q, K, V, self.shape, self.clusters(), self.routes(), self.compensate, O, self.workspace,
                           stream)

    def __call__(self, Q, K, V, O=None, stream=None):
        if O is None:
            O = self.torch.empty_like(Q)
        self.cluster(Q, K, stream)
        self.route(stream)
        self.attend(Q, K, V, O, stream)
        return O

    def forward_fused(self, Q, K, V, O, stream=None):
        """The whole path through the single ca_forward entry point."""
        if self.fwd_workspace is None:
            n = forward_workspace_bytes(self.shape, self.k)
            self.fwd_workspace = self.torch.empty(n, dtype=self.torch.uint8, device=Q.device)
        ca_forward(Q, K, V, self.shape, self.params, self.k, self.compensate, O, self.fwd_workspace, stream)
        return O

    def dense(self, Q, K, V, O, stream=None):
        ca_dense_attend(Q, K, V, self.shape, O, None, stream)
        return O
