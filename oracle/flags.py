"""ORACLE — test infrastructure only.  Literal flags.

Gzip-guided Sparse Attention (daiwk.github.io), section "核心公式", the r_i /
l_i equation: r_i = |gzip(x_{ib:(i+1)b})| / b, r̄ = (1/B) Σ_{j=1..B} r_j over
the B blocks of the sample, and l_i = 1[r_i > r̄].  "背景与主要改动" says the
threshold is the mean of the sample ("高于样本均值").

Written as that definition, in exact rational arithmetic (fractions.Fraction),
so no rounding can move a block across the threshold.  The comparison is
strict, so a sample whose blocks all have the same ratio has no literal block.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def literal_flags_row(lengths_row, b: int) -> np.ndarray:
    """l_i for one sample from its per-block gzip lengths (bytes)."""
    r = [Fraction(int(x), int(b)) for x in lengths_row]
    mean = sum(r, Fraction(0)) / len(r)
    return np.array([1 if ri > mean else 0 for ri in r], dtype=np.uint8)


def literal_flags(lengths: np.ndarray, b: int) -> np.ndarray:
    """Flags for every sample: lengths int [S, N] -> uint8 [S, N]."""
    lengths = np.asarray(lengths)
    if lengths.ndim == 1:
        return literal_flags_row(lengths, b)
    return np.stack([literal_flags_row(row, b) for row in lengths])
