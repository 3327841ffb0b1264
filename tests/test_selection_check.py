"""The adaptive-selection validity check the GPU tests fall back on at
numerical boundaries accepts the oracle's selections and rejects sets that
are not prefixes of the mass order, miss the target or are not minimal."""
import numpy as np
import pytest

from oracle import ca_oracle as orc
from tests.selection import adaptive_selection_problem


def _problem(seed, C=40, recall=0.9, min_count=4):
    rng = np.random.default_rng(seed)
    scores = rng.normal(0, 4.0, size=(6, C))
    count_k = rng.integers(1, 65, size=C)
    d = 64
    kept = orc.adaptive_route(scores, count_k, d, recall, min_count)
    W = orc.cluster_log_mass(scores, count_k, d)
    return kept, W, recall, min_count


@pytest.mark.parametrize("seed", range(4))
def test_oracle_selections_are_valid(seed):
    kept, W, recall, mc = _problem(seed)
    for a in range(len(kept)):
        assert adaptive_selection_problem(kept[a], W[a], recall, mc) is None


@pytest.mark.parametrize("seed", range(4))
def test_broken_selections_are_rejected(seed):
    kept, W, recall, mc = _problem(seed)
    for a in range(len(kept)):
        k = np.asarray(kept[a])
        order = np.lexsort((np.arange(W[a].size), -W[a]))
        rest = order[k.size:]
        if rest.size:
            # one cluster too many: not minimal (or, past the count, still a prefix)
            extra = np.append(k, rest[0])
            if k.size >= mc:
                assert "minimal" in adaptive_selection_problem(extra, W[a], recall, mc)
            # the heaviest kept cluster swapped for a dropped one: not a prefix
            swapped = np.append(np.setdiff1d(k, order[0]), rest[-1])
            assert adaptive_selection_problem(swapped, W[a], recall, mc) is not None
        if k.size > max(mc, 1):
            # the lightest kept cluster removed: misses the target
            short = np.setdiff1d(k, order[k.size - 1])
            assert "recall" in adaptive_selection_problem(short, W[a], recall, mc)
        assert adaptive_selection_problem(np.zeros(0, np.int64), W[a], recall, mc) == "empty selection"
