"""Pins for the oracle's literal flags and block mask (CPU only).

Flags: Gzip-guided Sparse Attention (daiwk.github.io), section "核心公式",
l_i = 1[r_i > r̄] with r̄ the mean over the sample's blocks.  Checked
against an integer restatement derived from it (multiply both sides by b*N),
against invariants that follow from the definition, and on special cases.

Mask: same section, M = M^lit ∪ M^local ∪ I with causality, and the edge
count O(L^2 + N w) for L literal blocks (the complexity equation).  Checked
against closed-form counts of live block pairs, brute force over every flag
vector of small samples, and the reductions the pages' definitions imply.
"""
import itertools

import numpy as np
import pytest

from oracle import flags as F
from oracle import mask as M

LOCAL, LITERAL, HYBRID = M.LOCAL, M.LITERAL, M.HYBRID


# ------------------------------------------------------------------ flags

def test_flags_integer_form():
    # r_i > mean  <=>  len_i / b > (1/N) Σ len_j / b  <=>  len_i * N > Σ len_j
    rng = np.random.default_rng(0)
    for _ in range(300):
        n = int(rng.integers(1, 80))
        b = int(rng.choice([16, 32, 64, 128]))
        ln = rng.integers(18, 18 + b + 5, size=n)
        want = (ln.astype(np.int64) * n > ln.sum()).astype(np.uint8)
        assert F.literal_flags_row(ln, b).tolist() == want.tolist()


def test_flags_equal_lengths_have_no_literal():
    assert F.literal_flags_row([40] * 17, 64).sum() == 0


def test_flags_never_all_literal():
    # at least one value is <= the mean, so at most N-1 blocks are literal
    rng = np.random.default_rng(1)
    for _ in range(500):
        ln = rng.integers(20, 90, size=int(rng.integers(1, 40)))
        assert F.literal_flags_row(ln, 64).sum() <= len(ln) - 1


def test_flags_single_outlier():
    ln = [30] * 10
    ln[7] = 31
    assert F.literal_flags_row(ln, 16).tolist() == [0] * 7 + [1] + [0] * 2


def test_flags_invariant_under_shift_and_scale():
    # adding the same constant (the 18 framing bytes) or scaling every
    # length by the same factor leaves the comparison with the mean intact
    rng = np.random.default_rng(2)
    for _ in range(200):
        ln = rng.integers(1, 100, size=int(rng.integers(2, 30)))
        base = F.literal_flags_row(ln, 64)
        assert (F.literal_flags_row(ln + 18, 64) == base).all()
        assert (F.literal_flags_row(ln * 3, 64) == base).all()
        assert (F.literal_flags_row(ln, 32) == base).all()


def test_flags_mean_is_per_sample():
    a = np.array([[10, 20, 30, 40], [100, 200, 300, 400]])
    assert F.literal_flags(a, 16).tolist() == [[0, 0, 1, 1], [0, 0, 1, 1]]


def test_flags_brute_force_rational():
    # exhaustive over small length vectors, comparing sums of ratios with
    # the mean by cross-multiplication in integers
    for n in range(1, 5):
        for ln in itertools.product(range(3), repeat=n):
            got = F.literal_flags_row(ln, 7).tolist()
            want = [1 if x * n > sum(ln) else 0 for x in ln]
            assert got == want


# ------------------------------------------------------------------- mask

def _local_count(n, w):
    return n * (w + 1) - w * (w + 1) // 2 if n > w else n * (n + 1) // 2


def _counts_closed_form(fl, w):
    fl = np.asarray(fl).astype(bool)
    n_blocks = len(fl)
    nl = int(fl.sum())
    local = _local_count(n_blocks, w)
    literal = nl * (nl + 1) // 2 + (n_blocks - nl)
    overlap = sum(1 for i in range(n_blocks) for j in range(i)
                  if i - j <= w and fl[i] and fl[j])
    hybrid = local + nl * (nl - 1) // 2 - overlap
    return local, literal, hybrid


def test_mask_closed_form_counts():
    rng = np.random.default_rng(3)
    for _ in range(300):
        n = int(rng.integers(1, 70))
        w = int(rng.integers(0, 6))
        fl = (rng.random(n) < rng.random()).astype(np.uint8)
        want = _counts_closed_form(fl, w)
        got = tuple(M.live_pairs(M.block_mask(fl, w, c)) for c in (LOCAL, LITERAL, HYBRID))
        assert got == want


def test_mask_edge_complexity_bound():
    # O(L^2 + N w): the hybrid count never exceeds L(L+1)/2 + N(w+1)
    rng = np.random.default_rng(4)
    for _ in range(200):
        n = int(rng.integers(1, 200))
        w = int(rng.integers(0, 8))
        fl = (rng.random(n) < 0.2).astype(np.uint8)
        nl = int(fl.sum())
        cnt = M.live_pairs(M.block_mask(fl, w, HYBRID))
        assert cnt <= nl * (nl + 1) // 2 + n * (w + 1)


def test_mask_sqrt_literals_is_linear():
    # with L ~ sqrt(N) literal blocks the live pairs grow about linearly in N
    ratios = []
    for n in (256, 1024, 4096):
        fl = np.zeros(n, dtype=np.uint8)
        fl[np.linspace(0, n - 1, int(np.sqrt(n))).astype(int)] = 1
        ratios.append(M.live_pairs(M.block_mask(fl, 4, HYBRID)) / n)
    assert max(ratios) < 1.6 * min(ratios)


@pytest.mark.parametrize("n", range(1, 9))
def test_mask_brute_force_small(n):
    # every flag vector of n blocks; live pairs listed pair by pair from the
    # definitions in words: same window, both literal, or the same block
    for bits in itertools.product((0, 1), repeat=n):
        for w in (0, 1, 2, n):
            for c in (LOCAL, LITERAL, HYBRID):
                m = M.block_mask(bits, w, c)
                for i in range(n):
                    for j in range(n):
                        in_window = i - w <= j <= i + w
                        both_literal = bits[i] == 1 and bits[j] == 1
                        same = i == j
                        live = {LOCAL: in_window, LITERAL: both_literal or same,
                                HYBRID: in_window or both_literal or same}[c]
                        assert m[i, j] == (live and j <= i)


def test_mask_all_literal_is_dense_causal():
    n = 23
    fl = np.ones(n, dtype=np.uint8)
    dense = np.tril(np.ones((n, n), dtype=bool))
    assert (M.block_mask(fl, 2, LITERAL) == dense).all()
    assert (M.block_mask(fl, 2, HYBRID) == dense).all()
    # ... and literal ∪ local ⊆ hybrid in general
    rng = np.random.default_rng(5)
    for _ in range(50):
        fl = (rng.random(n) < 0.5).astype(np.uint8)
        h = M.block_mask(fl, 2, HYBRID)
        assert ((M.block_mask(fl, 2, LITERAL) | M.block_mask(fl, 2, LOCAL)) == h).all()


def test_mask_wide_window_is_dense_causal():
    n = 19
    rng = np.random.default_rng(6)
    fl = (rng.random(n) < 0.3).astype(np.uint8)
    dense = np.tril(np.ones((n, n), dtype=bool))
    for w in (n - 1, n, 5 * n):
        assert (M.block_mask(fl, w, LOCAL) == dense).all()
        assert (M.block_mask(fl, w, HYBRID) == dense).all()


def test_mask_no_literal_blocks():
    n = 17
    fl = np.zeros(n, dtype=np.uint8)
    assert (M.block_mask(fl, 3, LITERAL) == np.eye(n, dtype=bool)).all()
    assert (M.block_mask(fl, 3, HYBRID) == M.block_mask(fl, 3, LOCAL)).all()


def test_row_and_col_lists_transpose():
    rng = np.random.default_rng(7)
    fl = (rng.random(40) < 0.4).astype(np.uint8)
    m = M.block_mask(fl, 2, HYBRID)
    rows = M.row_lists(m)
    cols = M.col_lists(m)
    pairs_r = {(i, int(j)) for i, r in enumerate(rows) for j in r}
    pairs_c = {(int(i), j) for j, c in enumerate(cols) for i in c}
    assert pairs_r == pairs_c
    assert all((np.diff(r) > 0).all() for r in rows)
    assert all((np.diff(c) > 0).all() for c in cols)


def test_token_pairs_count():
    rng = np.random.default_rng(8)
    fl = (rng.random(12) < 0.5).astype(np.uint8)
    for c in (LOCAL, LITERAL, HYBRID):
        m = M.block_mask(fl, 1, c)
        assert M.live_token_pairs(m, 4) == int(M.token_mask(m, 4).sum())
