"""Splitting one layer's heads across GPUs.

Every (batch, head) pair is clustered, routed and attended on its own
(ClusterAttention paper, Section 3.1: clustering runs "for each attention
head individually"), so one layer divides across GPUs by heads with no
collective on the data path. Rank r takes a contiguous range of the
flattened b * H + h indices; with head-major [B][H][N_alloc][d] tensors the
range is one contiguous block of memory, handed to the C ABI as a slice
(B = 1, H = the range's length) with ca_cluster_params.head_base = the
range's first index, which keys the random streams exactly as the
whole-layer call does.
"""
from __future__ import annotations

from typing import List, Tuple


def head_slices(n_heads: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous [begin, end) ranges of the flattened heads, one per rank;
    sizes differ by at most one (the first n_heads % world ranks take one more).
    A rank may get an empty range when world > n_heads."""
    if n_heads < 0 or world < 1:
        raise ValueError("n_heads >= 0 and world >= 1 required")
    base, extra = divmod(n_heads, world)
    out, b = [], 0
    for r in range(world):
        e = b + base + (1 if r < extra else 0)
        out.append((b, e))
        b = e
    return out


def rank_slice(n_heads: int, world: int, rank: int) -> Tuple[int, int]:
    """This rank's [begin, end) range of the flattened heads."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return head_slices(n_heads, world)[rank]
