"""ORACLE — test infrastructure only.  The adaptive block mask.

Gzip-guided Sparse Attention (daiwk.github.io), section "核心公式", the mask
equation: M = M^lit ∪ M^local ∪ I with M^lit_ij = 1[l_i = l_j = 1] and
M^local_ij = 1[|i - j| <= w], then intersected with the causal mask
("再与 causal mask 相交").  Section "背景与主要改动" splits the heads: 50% see only
the local window, 25% only the literal long-range edges, 25% the union of both.

Readings taken where the pages are silent:
  * local heads use M^local (which already holds the diagonal I);
  * literal heads use M^lit ∪ I, so a non-literal query block still attends
    to itself;
  * hybrid heads use the whole of M;
  * causality is applied to blocks here (j <= i) and to tokens inside the
    diagonal block by the attention (key token u <= query token t).
"""
from __future__ import annotations

import numpy as np

LOCAL, LITERAL, HYBRID = 0, 1, 2


def block_mask(flags_row, w: int, head_class: int) -> np.ndarray:
    """Boolean [N, N] block mask of one sample for one head class."""
    flags_row = np.asarray(flags_row).astype(bool)
    n = flags_row.shape[0]
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    m_lit = flags_row[:, None] & flags_row[None, :]
    m_local = np.abs(i - j) <= w
    ident = i == j
    causal = j <= i
    if head_class == LOCAL:
        m = m_local
    elif head_class == LITERAL:
        m = m_lit | ident
    elif head_class == HYBRID:
        m = m_lit | m_local | ident
    else:
        raise ValueError(f"unknown head class {head_class}")
    return m & causal


def row_lists(mask: np.ndarray) -> list[np.ndarray]:
    """Live key blocks of each query block, ascending."""
    return [np.nonzero(mask[i])[0].astype(np.int64) for i in range(mask.shape[0])]


def col_lists(mask: np.ndarray) -> list[np.ndarray]:
    """Query blocks that attend to each key block, ascending."""
    return [np.nonzero(mask[:, j])[0].astype(np.int64) for j in range(mask.shape[1])]


def token_mask(mask: np.ndarray, b: int) -> np.ndarray:
    """Token-level [N*b, N*b] mask: key u is visible to query t when their
    blocks are live in the block mask and u <= t."""
    n = mask.shape[0]
    t = np.arange(n * b)
    blk = t // b
    return mask[blk[:, None], blk[None, :]] & (t[None, :] <= t[:, None])


def live_pairs(mask: np.ndarray) -> int:
    """Number of live (query block, key block) pairs."""
    return int(mask.sum())


def live_token_pairs(mask: np.ndarray, b: int) -> int:
    """Number of (query token, key token) pairs attention computes: b*b per
    live off-diagonal block pair, b*(b+1)/2 per diagonal block."""
    diag = int(np.trace(mask))
    return (int(mask.sum()) - diag) * b * b + diag * b * (b + 1) // 2


# ------------------------------------------------ fixed comparison masks
#
# Fixed block masks the pages compare against: section "核心公式" (the
# background paragraph) names BigBird and Longformer as the content-blind
# baselines, and the arXiv abstract reports both at 8K context.  The pages
# give no definition, so the published patterns are read at block
# granularity, intersected with the causal mask like the adaptive one:
#   Longformer: sliding window of w blocks on each side plus g global blocks
#     (the first g); a global key block is seen by every later query block and
#     a global query block sees every earlier key block:
#     M_ij = 1[j <= i] * (1[i - j <= w] or 1[j < g] or 1[i < g]);
#   BigBird: the Longformer pattern plus r random key blocks per query block,
#     drawn causally: R_i = {u_ik mod (i + 1) : k < r} from r given uniform
#     32-bit words u_ik per query block (the random draws are inputs).

LONGFORMER, BIGBIRD = 0, 1


def fixed_block_mask(kind: int, n: int, w: int, g: int, rnd=None) -> np.ndarray:
    """Boolean [n, n] causal block mask of a fixed pattern.

    kind LONGFORMER or BIGBIRD; w window half-width in blocks, g global
    blocks; rnd uint32 [n, r] random words of one sample (BigBird only)."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    m = ((i - j) <= w) | (j < g) | (i < g)
    if kind == BIGBIRD:
        if rnd is None:
            raise ValueError("BigBird needs the random words")
        rnd = np.asarray(rnd, dtype=np.uint64).reshape(n, -1)
        for row in range(n):
            for u in rnd[row]:
                m[row, int(u % np.uint64(row + 1))] = True
    elif kind != LONGFORMER:
        raise ValueError(f"unknown fixed mask kind {kind}")
    return m & (j <= i)
