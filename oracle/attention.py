"""ORACLE — test infrastructure only.  Masked causal attention in float64.

Gzip-guided Sparse Attention (daiwk.github.io), section "复现边界": the
reproduction computes the dense score matrix and then applies the mask, i.e.
O = softmax(Q K^T / sqrt(d) + mask) V with -inf where the block mask of the
head's class (section "核心公式", mask equation) or causality forbids the pair.
The pages train the model (section "论文离线与线上效果": 20K steps), so the
gradient of that expression is part of the path as well.

Two forms of the same definition:
  * ``forward_dense`` / ``backward_dense`` build the token mask and run the
    dense masked softmax — the literal statement, for small inputs;
  * ``forward`` / ``backward`` visit, for each query block, only the key
    blocks its mask row lets it see (entries outside are exactly the -inf
    terms, which contribute nothing), so the large shapes finish.
Both work in float64 on float64 copies of the inputs.

Readings: the scale is 1/sqrt(d) (the pages do not state one); there is no
dropout, bias or key/value head sharing.  Every query row sees at least its
own token, so no row is empty.  LSE_t = m_t + ln Σ_u exp(s_tu - m_t), natural
logarithm.

Gradient (the chain rule through the softmax; P = softmax, D_t = Σ_e dO_te O_te):
    dV = P^T dO,  dP = dO V^T,  dS = P ∘ (dP - D),  dQ = scale · dS K,
    dK = scale · dS^T Q.
"""
from __future__ import annotations

import numpy as np

from .mask import block_mask, token_mask


def _f64(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _scale(d, scale):
    return 1.0 / np.sqrt(d) if not scale else float(scale)


# ---------------------------------------------------------------- dense form

def forward_dense(q, k, v, tmask, scale=None):
    """softmax(q k^T * scale + mask) v for one head.  q,k,v [T, d];
    tmask bool [T, T] (True = visible).  Returns (O [T, d], LSE [T])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    s = (q @ k.T) * _scale(q.shape[1], scale)
    s = np.where(tmask, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p / l) @ v
    return o, (m + np.log(l))[:, 0]


def backward_dense(q, k, v, do, tmask, scale=None):
    """Gradients (dQ, dK, dV) of the dense masked attention for one head."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    sc = _scale(q.shape[1], scale)
    s = np.where(tmask, (q @ k.T) * sc, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    p = p / p.sum(axis=1, keepdims=True)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    dd = (do * o).sum(axis=1, keepdims=True)
    ds = p * (dp - dd)
    return sc * ds @ k, sc * ds.T @ q, dv


# ------------------------------------------------------- block-visiting form

def _keys_of(mask_row, b, i):
    """Token indices of the key blocks live for query block i (ascending)."""
    blocks = np.nonzero(mask_row)[0]
    return (blocks[:, None] * b + np.arange(b)[None, :]).reshape(-1)


def _block_rows(q, k, v, mask, b, i, sc):
    """P, keys and O of query block i: P [b, nkeys] normalised, O [b, d]."""
    keys = _keys_of(mask[i], b, i)
    rows = np.arange(i * b, (i + 1) * b)
    s = (q[rows] @ k[keys].T) * sc
    s = np.where(keys[None, :] <= rows[:, None], s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    return p, keys, rows, p @ v[keys], (m + np.log(l))[:, 0]


def forward(q, k, v, mask, b, scale=None, q_blocks=None):
    """One head: q,k,v [T, d]; mask bool [N, N] block mask (causal).
    Returns O [T, d] and LSE [T] (rows of blocks not in q_blocks are NaN)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, d = q.shape
    sc = _scale(d, scale)
    o = np.full((T, v.shape[1]), np.nan)
    lse = np.full(T, np.nan)
    n = mask.shape[0]
    for i in (range(n) if q_blocks is None else q_blocks):
        _, _, rows, oi, li = _block_rows(q, k, v, mask, b, i, sc)
        o[rows] = oi
        lse[rows] = li
    return o, lse


def backward(q, k, v, do, mask, b, scale=None, q_blocks=None, k_blocks=None):
    """One head: gradients dQ, dK, dV [T, d] in float64.

    dQ is filled for the query blocks in q_blocks (all when None); dK and dV
    for the key blocks in k_blocks (all when None).  Rows outside are NaN.
    Every query block whose mask row reaches a requested key block is
    visited, since dK_u and dV_u sum over all rows t that see u.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    T, d = q.shape
    sc = _scale(d, scale)
    n = mask.shape[0]
    qb = set(range(n)) if q_blocks is None else set(int(x) for x in q_blocks)
    kb = set(range(n)) if k_blocks is None else set(int(x) for x in k_blocks)
    dq = np.full((T, d), np.nan)
    dk = np.full((T, d), np.nan)
    dv = np.full((T, v.shape[1]), np.nan)
    for j in kb:
        dk[j * b:(j + 1) * b] = 0.0
        dv[j * b:(j + 1) * b] = 0.0
    kb_arr = np.array(sorted(kb), dtype=np.int64)
    for i in range(n):
        need_q = i in qb
        need_k = kb_arr.size > 0 and bool(mask[i, kb_arr].any())
        if not (need_q or need_k):
            continue
        p, keys, rows, oi, _ = _block_rows(q, k, v, mask, b, i, sc)
        dp = do[rows] @ v[keys].T
        dd = (do[rows] * oi).sum(axis=1, keepdims=True)
        ds = p * (dp - dd)
        if need_q:
            dq[rows] = sc * ds @ k[keys]
        if need_k:
            sel = np.isin(keys // b, kb_arr)
            ks = keys[sel]
            dk[ks] += sc * ds[:, sel].T @ q[rows]
            dv[ks] += p[:, sel].T @ do[rows]
    return dq, dk, dv


# ------------------------------------------------------------ whole batches

def forward_batch(q, k, v, flags, w, head_classes, b, scale=None):
    """q,k,v [S, H, T, d]; flags [S, N]; head_classes [H].
    Returns O [S, H, T, d] and LSE [S, H, T] in float64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    S, H, T, d = q.shape
    o = np.empty((S, H, T, v.shape[3]))
    lse = np.empty((S, H, T))
    for s in range(S):
        masks = {c: block_mask(flags[s], w, c) for c in set(int(c) for c in head_classes)}
        for h in range(H):
            o[s, h], lse[s, h] = forward(q[s, h], k[s, h], v[s, h], masks[int(head_classes[h])], b, scale)
    return o, lse


def backward_batch(q, k, v, do, flags, w, head_classes, b, scale=None):
    """Gradients dQ, dK, dV [S, H, T, d] in float64 for whole batches."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    S, H, T, d = q.shape
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    for s in range(S):
        masks = {c: block_mask(flags[s], w, c) for c in set(int(c) for c in head_classes)}
        for h in range(H):
            dq[s, h], dk[s, h], dv[s, h] = backward(q[s, h], k[s, h], v[s, h], do[s, h],
                                                    masks[int(head_classes[h])], b, scale)
    return dq, dk, dv


def dense_token_mask(flags_row, w, head_class, b):
    """Token mask of one (sample, head class) — convenience for the dense form."""
    return token_mask(block_mask(flags_row, w, head_class), b)
