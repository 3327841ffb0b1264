"""Would the parity bar catch a plausible attention mistake?

Each mistake is planted in a copy of the oracle's compensated attention
(ClusterAttention paper, Section 3.1 and Appendix A eq. 21-22: softmax over
the kept key clusters' keys plus one term |b| e^{q . kbar_b / sqrt(d)} vbar_b
per excluded key cluster b), on the CPU, and run on the GPU parity tests' own
workloads with the oracle's clusters and routes. A mistake is caught when its
output differs from the correct one by more than the parity bounds
(tests/parity.py: max-abs or relative L2), which is what the GPU parity tests
assert of the kernels' output.

Mistakes:
  drop_block    the last kept key cluster of each query cluster is neither
                attended nor compensated (an off-by-one in the kept loop);
  remainder_c   every excluded cluster's weight uses ln c_k instead of
                ln |b|, wrong only for the ragged last cluster;
  bias_on_kept  the centroid terms cover the kept clusters too (the mask
                that removes a kept cluster's compensation is missing).
"""
import math

import numpy as np
import pytest

from oracle import ca_oracle as orc
from tests import parity
from tests.cases import CASES

MISTAKES = ["drop_block", "remainder_c", "bias_on_kept"]


def _planted(Q, K, V, h, kept, c, mistake):
    """The compensated attention of every query cluster, with one mistake."""
    d = Q.shape[1]
    scale = 1.0 / math.sqrt(d)
    Ck = h.count_k.shape[0]
    kmem = [h.perm_k[b * c: b * c + h.count_k[b]] for b in range(Ck)]
    kbar = np.stack([K[m].mean(axis=0) for m in kmem])
    vbar = np.stack([V[m].mean(axis=0) for m in kmem])
    counts = h.count_k.astype(np.float64)
    if mistake == "remainder_c":
        counts = np.full(Ck, float(c))
    logcnt = np.log(counts)
    O = np.zeros_like(Q)
    for a in range(h.count_q.shape[0]):
        qm = h.perm_q[a * c: a * c + h.count_q[a]]
        kept_a = np.asarray(kept[a], np.int64)
        attended = kept_a[:-1] if mistake == "drop_block" else kept_a
        J = np.concatenate([kmem[b] for b in attended]) if attended.size else np.zeros(0, np.int64)
        logits = (Q[qm] @ K[J].T) * scale
        vals = V[J]
        excl = np.setdiff1d(np.arange(Ck), kept_a)
        if mistake == "bias_on_kept":
            excl = np.arange(Ck)
        if excl.size:
            logits = np.concatenate([logits, (Q[qm] @ kbar[excl].T) * scale + logcnt[excl]], axis=1)
            vals = np.concatenate([vals, vbar[excl]], axis=0)
        w = np.exp(logits - logits.max(axis=1, keepdims=True))
        O[qm] = (w @ vals) / w.sum(axis=1, keepdims=True)
    return O


_cache = {}


def _head(name):
    """Workload, head-0 inputs in fp64, the oracle's clusters and top-k routes."""
    if name not in _cache:
        w = CASES[name]()
        Qf, Kf, Vf = (x[0, 0, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
        h = orc.cluster_head(Qf, Kf, w.c, seed=0, bh=0)
        kept = orc.topk_route(orc.centroid_scores(h.qbar, h.kbar), w.k)
        want = orc.compensated_attention(Qf, Kf, Vf, h.perm_q, h.count_q, h.perm_k, h.count_k, kept, w.c)
        _cache[name] = (w, Qf, Kf, Vf, h, kept, want)
    return _cache[name]


def _applies(mistake, w, h, kept):
    """Whether the mistake changes anything on this head at all."""
    Ck = h.count_k.shape[0]
    if mistake == "drop_block":
        # with one key cluster, dropping it leaves nothing to attend
        return Ck > 1
    if mistake == "remainder_c":
        ragged = np.flatnonzero(h.count_k != w.c)
        return any(r not in set(kept[a].tolist()) for r in ragged for a in range(len(kept)))
    return True


@pytest.mark.parametrize("name", list(CASES))
def test_copy_without_a_mistake_is_the_oracle(name):
    w, Qf, Kf, Vf, h, kept, want = _head(name)
    got = _planted(Qf, Kf, Vf, h, kept, w.c, None)
    assert np.abs(got - want).max() <= 1e-12


@pytest.mark.parametrize("mistake", MISTAKES)
@pytest.mark.parametrize("name", list(CASES))
def test_planted_mistake_exceeds_the_parity_bounds(name, mistake):
    w, Qf, Kf, Vf, h, kept, want = _head(name)
    if not _applies(mistake, w, h, kept):
        pytest.skip(f"{mistake} changes nothing on {name}")
    got = _planted(Qf, Kf, Vf, h, kept, w.c, mistake)
    max_abs, rel = parity.errors(got, want)
    assert max_abs > parity.MAX_ABS[w.dtype] or rel > parity.REL_L2[w.dtype], \
        f"{mistake} on {name}: max abs {max_abs:.3g}, rel-L2 {rel:.3g} would pass"
