"""Pins for the oracle's N:M mask: brute force over every n-subset of every
group on small inputs (ties constructed on purpose), and the invariants the
selection rule fixes (exactly n survivors, no dropped value above a kept one).
"""
import itertools
from fractions import Fraction

import numpy as np
import pytest


def _brute_force_group(v: np.ndarray, n: int):
    """Among the n-subsets with the largest exact sum of |v|, the one whose
    sorted index tuple is smallest: the n largest magnitudes, ties to the
    lower index."""
    best_key, best = None, None
    for sub in itertools.combinations(range(len(v)), n):
        s = sum(Fraction(abs(float(v[i]))) for i in sub)
        key = (-s, sub)
        if best_key is None or key < best_key:
            best_key, best = key, sub
    return best


NM = [(1, 2), (2, 4), (1, 4), (3, 4), (4, 8), (2, 8), (5, 8), (4, 4), (3, 16)]


@pytest.mark.parametrize("n,m", NM)
def test_mask_brute_force_with_ties(orc, n, m):
    rng = np.random.default_rng(n * 100 + m)
    rows, k = 6, 4 * m if m < 16 else 32
    # few distinct magnitudes and both signs of zero make ties common
    choices = np.float32([0.0, -0.0, 1.0, -1.0, 2.5, -2.5, 0.5, 7.0])
    x = rng.choice(choices, size=(rows, k)).astype(np.float32)
    x[0] = rng.standard_normal(k).astype(np.float32)
    idx, keep = orc.mask(x, n, m)
    for r in range(rows):
        for g in range(k // m):
            want = _brute_force_group(x[r, g * m:(g + 1) * m], n)
            assert tuple(int(i) for i in idx[r, g]) == want
            assert keep[r, g * m:(g + 1) * m].sum() == n


@pytest.mark.parametrize("n,m", [(2, 4), (4, 8)])
def test_mask_invariants_large(orc, n, m):
    x = np.random.default_rng(2).standard_normal((64, 1024)).astype(np.float32) ** 3
    idx, keep = orc.mask(x, n, m)
    a = np.abs(x).reshape(64, -1, m)
    kp = keep.reshape(64, -1, m).astype(bool)
    assert np.all(kp.sum(-1) == n)
    kept_min = np.where(kp, a, np.inf).min(-1)
    drop_max = np.where(~kp, a, -np.inf).max(-1)
    assert np.all(kept_min >= drop_max)
    assert np.all(np.diff(idx.astype(int), axis=-1) > 0)  # ascending, distinct
    # idx and keep describe the same set
    rebuilt = np.zeros_like(kp)
    np.put_along_axis(rebuilt, idx.astype(np.int64), True, axis=-1)
    assert np.array_equal(rebuilt, kp)
