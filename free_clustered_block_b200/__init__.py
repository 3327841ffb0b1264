"""ClusterAttention forward path on B200 (sm_100a).

Thin Python binding over libca (``include/ca.h``): the functions below only
marshal arguments (torch tensors -> device pointers and the current CUDA
stream) and call the C ABI of the same name. Every step of the computation
runs in the library's CUDA kernels; there is no Python or CPU compute path.
PyTorch supplies device memory and streams.

The library is built in-tree by ``python -m free_clustered_block_b200.build``
(or ``__graft_entry__.build()``); importing this package does not build it,
and calling into it without the built library raises ``LibraryMissing``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libca.so")

CA_OK, CA_ERR_INVALID_ARG, CA_ERR_UNSUPPORTED, CA_ERR_WORKSPACE, CA_ERR_CUDA, CA_ERR_TIMEOUT = range(6)
CA_BF16, CA_FP32 = 0, 1
CA_LAYOUT_BHND, CA_LAYOUT_BNHD = 0, 1

EXPORTED = [
    "ca_num_clusters", "ca_check_shape", "ca_cluster_workspace_bytes", "ca_attend_workspace_bytes",
    "ca_dense_workspace_bytes", "ca_forward_workspace_bytes", "ca_cluster", "ca_route", "ca_attend",
    "ca_dense_attend", "ca_forward", "ca_forward_host_workspace_bytes", "ca_forward_host",
    "ca_get_device_error", "ca_set_wait_limit", "ca_check_bounded_wait", "ca_status_string", "ca_version", "ca_launch_count",
    "ca_cluster_noalloc", "ca_route_adaptive", "ca_check_exp2_poly",
    "ca_attend_prepare", "ca_attend_prepared", "ca_num_key_clusters",
]


class LibraryMissing(RuntimeError):
    pass


class CAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class ca_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N_alloc", ctypes.c_int),
                ("n_valid", ctypes.c_int), ("d", ctypes.c_int), ("c", ctypes.c_int),
                ("dtype", ctypes.c_int), ("c_k", ctypes.c_int), ("layout", ctypes.c_int),
                ("H_total", ctypes.c_int)]


class ca_cluster_params(ctypes.Structure):
    _fields_ = [("power_iters", ctypes.c_int), ("sample_factor", ctypes.c_int),
                ("transform", ctypes.c_int), ("query_form", ctypes.c_int), ("seed", ctypes.c_uint64),
                ("method", ctypes.c_int), ("head_base", ctypes.c_int)]


class ca_clusters(ctypes.Structure):
    _fields_ = [("perm_q", ctypes.c_void_p), ("perm_k", ctypes.c_void_p), ("count_q", ctypes.c_void_p),
                ("count_k", ctypes.c_void_p), ("qbar", ctypes.c_void_p), ("kbar", ctypes.c_void_p)]


class ca_routes(ctypes.Structure):
    _fields_ = [("k", ctypes.c_int), ("kept_idx", ctypes.c_void_p), ("kept_bits", ctypes.c_void_p),
                ("kept_count", ctypes.c_void_p)]


_lib = None


def lib():
    """The loaded libca (ctypes.CDLL); raises LibraryMissing if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise LibraryMissing(f"{LIB_PATH} is not built: run `python -m free_clustered_block_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        vp, sz, i32, u64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_uint64
        sig = {
            "ca_num_clusters": (i32, [P(ca_shape)]),
            "ca_num_key_clusters": (i32, [P(ca_shape)]),
            "ca_check_shape": (i32, [P(ca_shape)]),
            "ca_cluster_workspace_bytes": (sz, [P(ca_shape)]),
            "ca_attend_workspace_bytes": (sz, [P(ca_shape)]),
            "ca_dense_workspace_bytes": (sz, [P(ca_shape)]),
            "ca_forward_workspace_bytes": (sz, [P(ca_shape), i32]),
            "ca_cluster": (i32, [vp, vp, P(ca_shape), P(ca_cluster_params), P(ca_clusters), vp, sz, vp]),
            "ca_route": (i32, [P(ca_shape), P(ca_clusters), P(ca_routes), vp]),
            "ca_attend": (i32, [vp, vp, vp, P(ca_shape), P(ca_clusters), P(ca_routes), i32, vp, vp, sz, vp]),
            "ca_dense_attend": (i32, [vp, vp, vp, P(ca_shape), vp, vp, sz, vp]),
            "ca_forward": (i32, [vp, vp, vp, P(ca_shape), P(ca_cluster_params), i32, i32, vp, vp, sz, vp]),
            "ca_forward_host_workspace_bytes": (sz, [P(ca_shape), i32]),
            "ca_forward_host": (i32, [vp, vp, vp, P(ca_shape), P(ca_cluster_params), i32, i32, vp, vp, sz, vp]),
            "ca_get_device_error": (i32, [vp]),
            "ca_set_wait_limit": (i32, [u64]),
            "ca_check_bounded_wait": (i32, [u64, i32, vp]),
            "ca_status_string": (ctypes.c_char_p, [i32]),
            "ca_version": (ctypes.c_char_p, []),
            "ca_launch_count": (i32, [P(ca_shape), i32]),
            "ca_cluster_noalloc": (i32, [vp, vp, P(ca_shape), P(ca_cluster_params), P(ca_clusters), vp]),
            "ca_route_adaptive": (i32, [P(ca_shape), P(ca_clusters), ctypes.c_double, i32, P(ca_routes), vp]),
            "ca_check_exp2_poly": (i32, [vp, vp, i32, vp]),
            "ca_attend_prepare": (i32, [vp, vp, vp, P(ca_shape), P(ca_clusters), vp, sz, vp]),
            "ca_attend_prepared": (i32, [vp, vp, vp, P(ca_shape), P(ca_clusters), P(ca_routes), i32, vp, vp, sz,
                                         vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    try:
        return lib().ca_status_string(status).decode()
    except LibraryMissing:
        return str(status)


def _check(status: int, where: str):
    if status != CA_OK:
        raise CAError(status, where)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def make_shape(B: int, H: int, N_alloc: int, n_valid: int, d: int, c: int, dtype: int, c_k: int = 0,
               layout: int = 0, H_total: int = 0) -> ca_shape:
    """c: query cluster size; c_k: key cluster size (0: the same as c).
    layout: CA_LAYOUT_BHND ([B, H, N, d]) or CA_LAYOUT_BNHD ([B, N, H_total, d],
    the call's heads first; H_total 0 means H)."""
    return ca_shape(B, H, N_alloc, n_valid, d, c, dtype, c_k, layout, H_total)


def make_params(power_iters: int = 8, sample_factor: int = 1, transform: int = 1,
                seed: int = 0, query_form: int = 0, method: int = 0, head_base: int = 0) -> ca_cluster_params:
    """query_form 0: queries as R_k q / |R_k q| (top-k selection, eq. 16);
    1: queries as R_k q (adaptive selection, eq. 15). method 0: recursive
    splitting; 1: random clusters (the error-analysis baseline); 2:
    diagonalized recursive splitting. head_base: global index of the call's
    first (b, h) pair, for a call on a slice of a layer's heads."""
    return ca_cluster_params(power_iters, sample_factor, transform, query_form, seed & ((1 << 64) - 1), method,
                             head_base)


def num_clusters(shape: ca_shape) -> int:
    """Query clusters C."""
    return lib().ca_num_clusters(ctypes.byref(shape))


def num_key_clusters(shape: ca_shape) -> int:
    """Key clusters C_k."""
    return lib().ca_num_key_clusters(ctypes.byref(shape))


def cluster_workspace_bytes(shape: ca_shape) -> int:
    return lib().ca_cluster_workspace_bytes(ctypes.byref(shape))


def attend_workspace_bytes(shape: ca_shape) -> int:
    return lib().ca_attend_workspace_bytes(ctypes.byref(shape))


def forward_workspace_bytes(shape: ca_shape, k: int) -> int:
    return lib().ca_forward_workspace_bytes(ctypes.byref(shape), k)


def forward_host_workspace_bytes(shape: ca_shape, k: int) -> int:
    return lib().ca_forward_host_workspace_bytes(ctypes.byref(shape), k)


def clusters_struct(perm_q, perm_k, count_q, count_k, qbar, kbar) -> ca_clusters:
    return ca_clusters(_ptr(perm_q), _ptr(perm_k), _ptr(count_q), _ptr(count_k), _ptr(qbar), _ptr(kbar))


def routes_struct(k: int, kept_idx, kept_bits, kept_count=None) -> ca_routes:
    return ca_routes(k, _ptr(kept_idx), _ptr(kept_bits), _ptr(kept_count))


def ca_cluster(Q, K, shape: ca_shape, params: Optional[ca_cluster_params], clusters: ca_clusters,
               workspace, stream=None):
    st = lib().ca_cluster(_ptr(Q), _ptr(K), ctypes.byref(shape),
                          ctypes.byref(params) if params is not None else None,
                          ctypes.byref(clusters), _ptr(workspace),
                          0 if workspace is None else workspace.numel() * workspace.element_size(),
                          _stream(stream))
    _check(st, "ca_cluster")


def ca_cluster_noalloc(Q, K, shape: ca_shape, params: Optional[ca_cluster_params], clusters: ca_clusters,
                       stream=None):
    """ca_cluster with the library's fixed 16 MiB device scratch instead of a
    workspace, for callers that cannot allocate device memory."""
    st = lib().ca_cluster_noalloc(_ptr(Q), _ptr(K), ctypes.byref(shape),
                                  ctypes.byref(params) if params is not None else None,
                                  ctypes.byref(clusters), _stream(stream))
    _check(st, "ca_cluster_noalloc")


def ca_route(shape: ca_shape, centroids: ca_clusters, routes: ca_routes, stream=None):
    _check(lib().ca_route(ctypes.byref(shape), ctypes.byref(centroids), ctypes.byref(routes),
                          _stream(stream)), "ca_route")


def ca_route_adaptive(shape: ca_shape, centroids: ca_clusters, recall: float, min_count: int,
                      routes: ca_routes, stream=None):
    """Adaptive selection: per query cluster, key clusters by decreasing
    estimated attention mass until `recall` of the total, at least
    `min_count`; routes.kept_count receives the counts."""
    _check(lib().ca_route_adaptive(ctypes.byref(shape), ctypes.byref(centroids), float(recall), int(min_count),
                                   ctypes.byref(routes), _stream(stream)), "ca_route_adaptive")


def ca_attend(Q, K, V, shape: ca_shape, clusters: ca_clusters, routes: ca_routes, compensate: bool, O,
              workspace, stream=None):
    st = lib().ca_attend(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shape), ctypes.byref(clusters),
                         ctypes.byref(routes), int(bool(compensate)), _ptr(O), _ptr(workspace),
                         0 if workspace is None else workspace.numel() * workspace.element_size(),
                         _stream(stream))
    _check(st, "ca_attend")


def ca_attend_prepare(Q, K, V, shape: ca_shape, clusters: ca_clusters, workspace, stream=None):
    """First half of ca_attend: value centroids and the cluster-ordered copies into the workspace."""
    st = lib().ca_attend_prepare(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shape), ctypes.byref(clusters),
                                 _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
                                 _stream(stream))
    _check(st, "ca_attend_prepare")


def ca_attend_prepared(Q, K, V, shape: ca_shape, clusters: ca_clusters, routes: ca_routes, compensate: bool, O,
                       workspace, stream=None):
    """Second half of ca_attend: the attention kernel, from a prepared workspace."""
    st = lib().ca_attend_prepared(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shape), ctypes.byref(clusters),
                                  ctypes.byref(routes), int(bool(compensate)), _ptr(O), _ptr(workspace),
                                  0 if workspace is None else workspace.numel() * workspace.element_size(),
                                  _stream(stream))
    _check(st, "ca_attend_prepared")


def ca_dense_attend(Q, K, V, shape: ca_shape, O, workspace=None, stream=None):
    st = lib().ca_dense_attend(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shape), _ptr(O), _ptr(workspace),
                               0 if workspace is None else workspace.numel() * workspace.element_size(),
                               _stream(stream))
    _check(st, "ca_dense_attend")


def ca_forward(Q, K, V, shape: ca_shape, params: Optional[ca_cluster_params], k: int, compensate: bool, O,
               workspace, stream=None):
    st = lib().ca_forward(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(shape),
                          ctypes.byref(params) if params is not None else None, k, int(bool(compensate)),
                          _ptr(O), _ptr(workspace), workspace.numel() * workspace.element_size(),
                          _stream(stream))
    _check(st, "ca_forward")


def ca_forward_host(Qh, Kh, Vh, shape: ca_shape, params: Optional[ca_cluster_params], k: int,
                    compensate: bool, Oh, workspace, stream=None):
    """Host (CPU, ideally pinned) tensors in and out; copies run inside the call."""
    st = lib().ca_forward_host(_ptr(Qh), _ptr(Kh), _ptr(Vh), ctypes.byref(shape),
                               ctypes.byref(params) if params is not None else None, k,
                               int(bool(compensate)), _ptr(Oh), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "ca_forward_host")


def ca_get_device_error(stream=None) -> int:
    return lib().ca_get_device_error(_stream(stream))


def ca_set_wait_limit(limit_ns: int):
    _check(lib().ca_set_wait_limit(limit_ns), "ca_set_wait_limit")


def ca_check_bounded_wait(limit_ns: int, arrive: bool, stream=None) -> int:
    return lib().ca_check_bounded_wait(limit_ns, 1 if arrive else 0, _stream(stream))


def ca_check_exp2_poly(x, y, stream=None):
    """y[i] = the attention kernel's FMA-pipe evaluation of 2^x[i] (device fp32 tensors)."""
    _check(lib().ca_check_exp2_poly(_ptr(x), _ptr(y), int(x.numel()), _stream(stream)), "ca_check_exp2_poly")


def launch_count(shape: ca_shape, stage: int) -> int:
    """Kernel launches per call: stage 0 cluster, 1 route, 2 attend, 3 dense."""
    return lib().ca_launch_count(ctypes.byref(shape), stage)


def version() -> str:
    return lib().ca_version().decode()


from .layer import ClusterAttention  # noqa: E402,F401
