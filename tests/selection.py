"""Validity of an adaptive selection when it may legitimately differ from the
oracle's (ClusterAttention paper, Section 3.3.2 "Selection", second method:
key clusters in decreasing estimated mass until the kept mass reaches the
recall fraction of the total, and at least the minimum count).

At a numerical boundary (the running mass within 1e-12 of the target, or two
masses tied within 1e-12) the GPU and the oracle may round the fp64
exponentials and sums differently; the GPU's set must then still be a valid
and minimal greedy selection.
"""
import numpy as np


def adaptive_selection_problem(got, W, recall, min_count, rel=1e-12):
    """None if ``got`` (kept key clusters) is a valid, minimal greedy selection
    for log-masses ``W``; otherwise a description of what is wrong."""
    got = np.asarray(got, np.int64)
    W = np.asarray(W, np.float64)
    m = np.exp(W - W.max())
    total = m.sum()
    tie = rel * max(1.0, abs(W).max())
    if got.size == 0:
        return "empty selection"
    if np.unique(got).size != got.size:
        return "repeated cluster"
    dropped = np.setdiff1d(np.arange(W.size), got)
    if dropped.size and W[got].min() < W[dropped].max() - tie:
        return "not a prefix of the mass order"
    if got.size < min(min_count, W.size):
        return "fewer clusters than the minimum count"
    if m[got].sum() < recall * total * (1 - rel):
        return "kept mass below the recall target"
    if got.size > min(min_count, W.size):
        lightest = got[np.argmin(W[got])]
        if m[got].sum() - m[lightest] >= recall * total * (1 + rel):
            return "not minimal: the target is met without the lightest kept cluster"
    return None
