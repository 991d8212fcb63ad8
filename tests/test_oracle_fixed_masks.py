"""The oracle's fixed comparison masks (Longformer, BigBird at block
granularity) against facts that do not come from it: the adaptive mask's
local class (Longformer without global blocks is the sliding window), the
dense causal triangle, closed-form row and column counts, a mask worked out
by hand, and invariants of the random picks."""
import numpy as np
import pytest

from oracle import mask as om



def _tril(n):
    return np.tril(np.ones((n, n), dtype=bool))


@pytest.mark.parametrize("n,w", [(1, 0), (7, 0), (7, 2), (16, 3), (33, 40)])
def test_longformer_without_globals_is_the_local_window(n, w):
    flags = np.zeros(n, dtype=np.uint8)
    want = om.block_mask(flags, w, om.LOCAL)
    assert np.array_equal(om.fixed_block_mask(om.LONGFORMER, n, w, 0), want)


@pytest.mark.parametrize("n,w,g", [(5, 0, 5), (9, 1, 9), (9, 0, 20)])
def test_all_global_is_dense_causal(n, w, g):
    assert np.array_equal(om.fixed_block_mask(om.LONGFORMER, n, w, g), _tril(n))


@pytest.mark.parametrize("n,w,g", [(1, 0, 0), (12, 0, 1), (12, 2, 3), (40, 5, 2), (40, 50, 1), (64, 1, 0)])
def test_longformer_counts_closed_form(n, w, g):
    m = om.fixed_block_mask(om.LONGFORMER, n, w, g)
    for i in range(n):
        # window [max(0, i-w), i] plus the globals left of it
        want = min(i, w) + 1 + min(g, max(0, i - w))
        assert m[i].sum() == want, i
    for j in range(n):
        # window [j, min(n-1, j+w)], every later row when j is global
        want = (n - j) if j < g else (min(n - 1, j + w) - j + 1)
        assert m[:, j].sum() == want, j


def test_bigbird_by_hand():
    # n = 6, w = 1, g = 1, r = 2; picks u mod (i + 1):
    #   row 0: 0, 0        row 1: 1, 0        row 2: 9 % 3 = 0, 5 % 3 = 2
    #   row 3: 7 % 4 = 3, 10 % 4 = 2   row 4: 13 % 5 = 3, 2   row 5: 17 % 6 = 5, 6 % 6 = 0
    rnd = np.array([[4, 8], [3, 2], [9, 5], [7, 10], [13, 2], [17, 6]], dtype=np.uint32)
    want = np.array([
        [1, 0, 0, 0, 0, 0],
        [1, 1, 0, 0, 0, 0],
        [1, 1, 1, 0, 0, 0],
        [1, 0, 1, 1, 0, 0],
        [1, 0, 1, 1, 1, 0],
        [1, 0, 0, 0, 1, 1],
    ], dtype=bool)
    assert np.array_equal(om.fixed_block_mask(om.BIGBIRD, 6, 1, 1, rnd), want)


def test_bigbird_without_random_blocks_is_longformer():
    rnd = np.zeros((20, 0), dtype=np.uint32)
    assert np.array_equal(om.fixed_block_mask(om.BIGBIRD, 20, 2, 1, rnd),
                          om.fixed_block_mask(om.LONGFORMER, 20, 2, 1))


@pytest.mark.parametrize("n,w,g,r", [(10, 0, 0, 1), (50, 1, 2, 3), (128, 1, 2, 8)])
def test_bigbird_invariants(n, w, g, r):
    rnd = np.random.default_rng(n + r).integers(0, 2**32, size=(n, r), dtype=np.uint64).astype(np.uint32)
    m = om.fixed_block_mask(om.BIGBIRD, n, w, g, rnd)
    base = om.fixed_block_mask(om.LONGFORMER, n, w, g)
    assert not (m & ~_tril(n)).any()            # causal
    assert (m | base).sum() == m.sum()          # holds the Longformer pattern
    extra = m & ~base
    for i in range(n):
        picks = {int(u) % (i + 1) for u in rnd[i]}
        assert set(np.nonzero(extra[i])[0].tolist()) == picks - set(np.nonzero(base[i])[0].tolist())
        assert m[i].sum() <= base[i].sum() + r
