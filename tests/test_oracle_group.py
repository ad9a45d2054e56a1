"""Pins of the oracle's group entropy-bounded accept (the longest prefix of a
canvas's positions, ordered by entropy, whose cumulative entropy is within the
bound).

Independent characterisation used by the brute force: the accepted set is a set
of positions of largest size whose entropies sum to at most the bound; among those
it has the least total, and among equal totals the smallest positions.  Entropies
are multiples of 1/64 in the brute force, so every sum is exact.
"""

import itertools

import numpy as np
import pytest

from oracle import stage


def _brute(H, bound):
    n = len(H)
    best = None
    for r in range(n, -1, -1):
        for sub in itertools.combinations(range(n), r):
            tot = sum(H[i] for i in sub)
            if tot <= bound:
                key = (tot, tuple(sorted(sorted(sub), key=lambda i: (H[i], i))))
                if best is None or key < best[0]:
                    best = (key, set(sub))
        if best is not None:
            return best[1]
    return set()


@pytest.mark.parametrize("seed", range(12))
def test_group_accept_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 10))
    H = rng.integers(0, 24, size=n) / 64.0                # ties and zeros occur
    bound = float(rng.integers(0, 40)) / 64.0
    kept = np.arange(100, 100 + n)
    ren = np.arange(200, 200 + n)
    tok, acc, _, _ = stage.group_accept(H, kept, bound, ren)
    want = _brute(list(H), bound)
    assert set(np.nonzero(acc)[0].tolist()) == want
    assert np.array_equal(tok, np.where(acc == 1, kept, ren))


def test_closed_forms():
    kept, ren = np.arange(8), np.arange(8) + 50
    # all zero entropies: everything fits
    _, acc, _, _ = stage.group_accept(np.zeros(8), kept, 0.1, ren)
    assert acc.all()
    # every entropy above the bound: nothing is accepted (no forced progress)
    _, acc, _, _ = stage.group_accept(np.full(8, 0.2), kept, 0.1, ren)
    assert not acc.any()
    # three equal entropies of 0.05 with bound 0.1: the two lowest positions
    _, acc, cm, og = stage.group_accept(np.array([0.3, 0.05, 0.05, 0.05]), np.arange(4), 0.1, np.arange(4) + 9)
    assert acc.tolist() == [0, 1, 1, 0] and og == 0.0 and cm == pytest.approx(0.0, abs=1e-15)
    # a tiny negative entropy (rounding) counts as zero
    _, acc, _, _ = stage.group_accept(np.array([-1e-9, 0.2]), np.arange(2), 0.1, np.arange(2) + 5)
    assert acc.tolist() == [1, 0]


def test_subset_of_per_position_rule_and_permutation():
    rng = np.random.default_rng(7)
    H = rng.exponential(0.01, size=256)
    H[rng.choice(256, 40, replace=False)] = rng.uniform(0.2, 5.0, 40)
    kept, ren = np.arange(256), np.arange(256) + 1000
    _, acc, _, _ = stage.group_accept(H, kept, 0.1, ren)
    _, acc_pos = stage.eb_accept(H, kept, 0.1, ren)
    assert acc.sum() > 0 and np.all(acc <= acc_pos)                    # every accepted H is <= the bound
    assert H[acc == 1].sum() <= 0.1 < H[acc == 1].sum() + H[acc == 0].min()
    perm = rng.permutation(256)                                        # distinct entropies: equivariant
    _, acc_p, _, _ = stage.group_accept(H[perm], kept, 0.1, ren)
    assert np.array_equal(acc_p, acc[perm])
