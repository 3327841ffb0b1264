"""The C-ABI library loads, exports every entry point include/ca.h declares,
and validates arguments on the host (no GPU needed: every call below is
rejected before any launch)."""
import ctypes
import os
import re

import pytest

import free_clustered_block_b200 as ca
from oracle import ca_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from free_clustered_block_b200 import build
    build.build()   # incremental: rebuilds only what changed
    return ca.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "ca.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ca_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 15
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(ca.EXPORTED)


def test_version_and_status_strings(lib):
    assert "sm_100a" in ca.version()
    assert ca.status_string(ca.CA_ERR_WORKSPACE) == "CA_ERR_WORKSPACE"


@pytest.mark.parametrize("n,c", [(1024, 64), (75600, 128), (65536, 128), (262144, 256), (100, 128), (1000, 64)])
def test_num_clusters_matches_tree_rule(lib, n, c):
    s = ca.make_shape(1, 2, n, n, 64, c, ca.CA_BF16)
    assert ca.num_clusters(s) == orc.num_clusters(n, c)
    assert ca.cluster_workspace_bytes(s) > 0
    assert ca.attend_workspace_bytes(s) > 0


def test_shape_validation(lib):
    ok = ca.make_shape(1, 1, 1024, 1024, 64, 64, ca.CA_FP32)
    assert lib.ca_check_shape(ctypes.byref(ok)) == ca.CA_OK
    bad = [
        (ca.make_shape(1, 1, 1024, 1024, 96, 64, ca.CA_FP32), ca.CA_ERR_UNSUPPORTED),   # d
        (ca.make_shape(1, 1, 1024, 1024, 64, 100, ca.CA_FP32), ca.CA_ERR_UNSUPPORTED),  # c
        (ca.make_shape(1, 1, 1000, 1024, 64, 64, ca.CA_FP32), ca.CA_ERR_INVALID_ARG),   # n > N_alloc
        (ca.make_shape(0, 1, 1024, 1024, 64, 64, ca.CA_FP32), ca.CA_ERR_INVALID_ARG),   # B
        (ca.make_shape(1, 1, 1024, 0, 64, 64, ca.CA_FP32), ca.CA_ERR_INVALID_ARG),      # empty
        (ca.make_shape(1, 1, 1024, 1024, 64, 64, 7), ca.CA_ERR_INVALID_ARG),            # dtype
        (ca.make_shape(1, 2, 1024, 1024, 64, 64, ca.CA_FP32, layout=2), ca.CA_ERR_INVALID_ARG),       # layout
        (ca.make_shape(1, 2, 1024, 1024, 64, 64, ca.CA_FP32, layout=ca.CA_LAYOUT_BHND, H_total=3),
         ca.CA_ERR_INVALID_ARG),                                                                      # BHND H_total
        (ca.make_shape(1, 2, 1024, 1024, 64, 64, ca.CA_FP32, layout=ca.CA_LAYOUT_BNHD, H_total=1),
         ca.CA_ERR_INVALID_ARG),                                                                      # H_total < H
    ]
    for s, want in bad:
        assert lib.ca_check_shape(ctypes.byref(s)) == want
        assert lib.ca_num_clusters(ctypes.byref(s)) == -1
    # token-major: a slice of heads (H_total > H) is a valid shape, but the
    # host-buffer forward needs the buffers to hold exactly the call's heads
    sl = ca.make_shape(1, 2, 1024, 1024, 64, 64, ca.CA_BF16, layout=ca.CA_LAYOUT_BNHD, H_total=4)
    assert lib.ca_check_shape(ctypes.byref(sl)) == ca.CA_OK
    assert ca.forward_host_workspace_bytes(sl, 4) == 0
    full = ca.make_shape(1, 4, 1024, 1024, 64, 64, ca.CA_BF16, layout=ca.CA_LAYOUT_BNHD)
    assert ca.forward_host_workspace_bytes(full, 4) > 0


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_calls_are_rejected_before_launch(lib):
    s = ca.make_shape(1, 1, 1024, 1024, 64, 64, ca.CA_FP32)
    A = 0x10000
    cl = ca.ca_clusters(A, A, A, A, A, A)
    rt = ca.ca_routes(4, A, A)
    need = ca.cluster_workspace_bytes(s)
    # workspace too small
    assert lib.ca_cluster(_fake(A), _fake(A), ctypes.byref(s), None, ctypes.byref(cl), _fake(A), need - 1,
                          None) == ca.CA_ERR_WORKSPACE
    # null input
    assert lib.ca_cluster(None, _fake(A), ctypes.byref(s), None, ctypes.byref(cl), _fake(A), need,
                          None) == ca.CA_ERR_INVALID_ARG
    # misaligned input
    assert lib.ca_cluster(_fake(A + 4), _fake(A), ctypes.byref(s), None, ctypes.byref(cl), _fake(A), need,
                          None) == ca.CA_ERR_INVALID_ARG
    # bad params
    p = ca.make_params(power_iters=-1)
    assert lib.ca_cluster(_fake(A), _fake(A), ctypes.byref(s), ctypes.byref(p), ctypes.byref(cl), _fake(A),
                          need, None) == ca.CA_ERR_INVALID_ARG
    # method out of range; diagonalized splitting takes only the sample factor a = 1
    for bad, want in ((ca.make_params(method=3), ca.CA_ERR_INVALID_ARG),
                      (ca.make_params(method=-1), ca.CA_ERR_INVALID_ARG),
                      (ca.make_params(method=2, sample_factor=2), ca.CA_ERR_UNSUPPORTED),
                      (ca.make_params(query_form=2), ca.CA_ERR_INVALID_ARG)):
        assert lib.ca_cluster(_fake(A), _fake(A), ctypes.byref(s), ctypes.byref(bad), ctypes.byref(cl),
                              _fake(A), need, None) == want
    # the bounded-wait check rejects a zero or over-long limit before launching
    assert lib.ca_check_bounded_wait(0, 0, None) == ca.CA_ERR_INVALID_ARG
    assert lib.ca_check_bounded_wait(20_000_000_000, 0, None) == ca.CA_ERR_INVALID_ARG
    # k out of range
    for k in (0, 17):
        r = ca.ca_routes(k, A, A)
        assert lib.ca_route(ctypes.byref(s), ctypes.byref(cl), ctypes.byref(r), None) == ca.CA_ERR_INVALID_ARG
    # attend: workspace too small, null O
    aneed = ca.attend_workspace_bytes(s)
    assert lib.ca_attend(_fake(A), _fake(A), _fake(A), ctypes.byref(s), ctypes.byref(cl), ctypes.byref(rt), 1,
                         _fake(A), _fake(A), aneed - 1, None) == ca.CA_ERR_WORKSPACE
    assert lib.ca_attend(_fake(A), _fake(A), _fake(A), ctypes.byref(s), ctypes.byref(cl), ctypes.byref(rt), 1,
                         None, _fake(A), aneed, None) == ca.CA_ERR_INVALID_ARG
    # forward: k out of range -> no workspace size
    assert ca.forward_workspace_bytes(s, 0) == 0
    assert ca.forward_workspace_bytes(s, 17) == 0
    assert ca.forward_workspace_bytes(s, 4) > 0
    # unsupported head dim anywhere
    s96 = ca.make_shape(1, 1, 1024, 1024, 96, 64, ca.CA_FP32)
    assert lib.ca_dense_attend(_fake(A), _fake(A), _fake(A), ctypes.byref(s96), _fake(A), None, 0,
                               None) == ca.CA_ERR_UNSUPPORTED


def test_noalloc_scratch_covers_its_stated_examples(lib):
    # the allocation-free clustering entry promises room for two 65,536-token
    # heads at d = 64 or one 75,600-token head at d = 128 in its 16 MiB
    for args in ((1, 2, 65536, 65536, 64, 128), (1, 1, 76800, 75600, 128, 128)):
        s = ca.make_shape(*args, ca.CA_BF16)
        assert 0 < ca.cluster_workspace_bytes(s) <= 16 << 20


def test_wait_limit_setter_rejects_limits_above_ten_seconds(lib):
    assert lib.ca_set_wait_limit(10_000_000_001) == ca.CA_ERR_INVALID_ARG
    assert lib.ca_set_wait_limit(2**64 - 1) == ca.CA_ERR_INVALID_ARG
    assert lib.ca_set_wait_limit(5_000_000) == ca.CA_OK
    assert lib.ca_set_wait_limit(0) == ca.CA_OK          # back to the default
    assert lib.ca_check_exp2_poly(None, None, 4, None) == ca.CA_ERR_INVALID_ARG
