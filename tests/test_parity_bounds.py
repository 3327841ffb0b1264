"""The relative-L2 bound for bf16 attention (tests/parity.py), checked against
a model of the kernel's roundings on the parity workloads.

The model takes the oracle's compensated attention (ClusterAttention paper,
Section 3.1 and Appendix A eq. 21-22) in fp64 and applies the two roundings
the derivation names: the weights P to bf16 before the P V sums, and the
output O to bf16 at the store (the row sums use the unrounded weights, as the
kernel keeps them in fp32 registers). Its error must sit where the
derivation puts it (about 2.3e-3, between one rounding's RMS and the bound).
"""
import numpy as np
import pytest

from oracle import ca_oracle as orc
from tests import parity
from tests.cases import CASES


def _bf16(x):
    """Round to the nearest bf16 (ties to even), returned as float64."""
    f = np.asarray(x, np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


def test_bf16_rounding_model():
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -9, -2.5, 1e-3])
    y = _bf16(x)
    assert y[0] == 1.0 and y[1] == 1.0          # a tie goes to the even mantissa
    assert y[2] == 1.0 + 2.0 ** -7              # above the tie rounds up
    assert y[3] == -2.5
    assert abs(y[4] / 1e-3 - 1) <= 2.0 ** -8


def _model(Q, K, V, h, kept, c):
    """Compensated attention with P and O rounded to bf16 (fp64 otherwise)."""
    d = Q.shape[1]
    Ck = h.count_k.shape[0]
    kmem = [h.perm_k[b * c: b * c + h.count_k[b]] for b in range(Ck)]
    kbar = np.stack([K[m].mean(axis=0) for m in kmem])
    vbar = np.stack([V[m].mean(axis=0) for m in kmem])
    logcnt = np.log(h.count_k.astype(np.float64))
    O = np.zeros_like(Q)
    for a in range(h.count_q.shape[0]):
        qm = h.perm_q[a * c: a * c + h.count_q[a]]
        kept_a = np.asarray(kept[a], np.int64)
        J = np.concatenate([kmem[b] for b in kept_a])
        logits = Q[qm] @ K[J].T / np.sqrt(d)
        vals = V[J]
        excl = np.setdiff1d(np.arange(Ck), kept_a)
        if excl.size:
            logits = np.concatenate([logits, Q[qm] @ kbar[excl].T / np.sqrt(d) + logcnt[excl]], axis=1)
            vals = np.concatenate([vals, vbar[excl]], axis=0)
        w = np.exp(logits - logits.max(axis=1, keepdims=True))
        O[qm] = _bf16((_bf16(w) @ vals) / w.sum(axis=1, keepdims=True))
    return O


@pytest.mark.parametrize("name", list(CASES))
def test_rounding_model_error_is_inside_the_bound(name):
    w = CASES[name]()
    if w.dtype != "bf16":
        pytest.skip("fp32 case")
    Qf, Kf, Vf = (x[0, 0, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
    h = orc.cluster_head(Qf, Kf, w.c, seed=0, bh=0)
    kept = orc.topk_route(orc.centroid_scores(h.qbar, h.kbar), w.k)
    exact = orc.compensated_attention(Qf, Kf, Vf, h.perm_q, h.count_q, h.perm_k, h.count_k, kept, w.c)
    model = _model(Qf, Kf, Vf, h, kept, w.c)
    max_abs, rel = parity.errors(model, exact)
    # one bf16 rounding of O alone has an RMS relative error of about 2^-8 / sqrt(3)
    # (mantissas spread over [1, 2) lower it somewhat); P's roundings add little
    assert 1.0e-3 <= rel <= 3.3e-3, f"{name}: model rel-L2 {rel:.3g}"
    assert rel <= parity.REL_L2["bf16"] / 3
    assert max_abs <= parity.MAX_ABS["bf16"]


def _model_fp32(Q, K, V, h, kept, c):
    """Compensated attention with every operation in fp32 (the SIMT kernel's precision)."""
    f = np.float32
    d = Q.shape[1]
    Q32, K32, V32 = Q.astype(f), K.astype(f), V.astype(f)
    Ck = h.count_k.shape[0]
    kmem = [h.perm_k[b * c: b * c + h.count_k[b]] for b in range(Ck)]
    kbar = np.stack([K[m].mean(axis=0) for m in kmem]).astype(f)   # centroids arrive from fp64
    vbar = np.stack([V[m].mean(axis=0) for m in kmem]).astype(f)
    logcnt = np.log(h.count_k.astype(f))
    sc = f(1.0 / np.sqrt(d))
    O = np.zeros(Q.shape, f)
    for a in range(h.count_q.shape[0]):
        qm = h.perm_q[a * c: a * c + h.count_q[a]]
        kept_a = np.asarray(kept[a], np.int64)
        J = np.concatenate([kmem[b] for b in kept_a])
        logits = (Q32[qm] @ K32[J].T) * sc
        vals = V32[J]
        excl = np.setdiff1d(np.arange(Ck), kept_a)
        if excl.size:
            logits = np.concatenate([logits, (Q32[qm] @ kbar[excl].T) * sc + logcnt[excl]], axis=1)
            vals = np.concatenate([vals, vbar[excl]], axis=0)
        w = np.exp(logits - logits.max(axis=1, keepdims=True))
        O[qm] = (w @ vals) / w.sum(axis=1, keepdims=True)
    return O.astype(np.float64)


@pytest.mark.parametrize("name", list(CASES))
def test_fp32_model_error_is_inside_the_bound(name):
    w = CASES[name]()
    if w.dtype != "fp32":
        pytest.skip("bf16 case")
    Qf, Kf, Vf = (x[0, 0, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
    h = orc.cluster_head(Qf, Kf, w.c, seed=0, bh=0)
    kept = orc.topk_route(orc.centroid_scores(h.qbar, h.kbar), w.k)
    exact = orc.compensated_attention(Qf, Kf, Vf, h.perm_q, h.count_q, h.perm_k, h.count_k, kept, w.c)
    max_abs, rel = parity.errors(_model_fp32(Qf, Kf, Vf, h, kept, w.c), exact)
    # the derivation's estimate is ~5e-6; the bound leaves a factor of four
    assert rel <= parity.REL_L2["fp32"] / 4, f"{name}: model rel-L2 {rel:.3g}"
    assert max_abs <= parity.MAX_ABS["fp32"]
