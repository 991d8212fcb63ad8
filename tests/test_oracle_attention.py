"""Pins for the oracle's masked attention and its gradient (CPU only).

The attention arithmetic is checked against torch's scaled_dot_product_attention
(math kernel, float64) and autograd through it, independent routines that
take the mask as given; the mask/attention combination against the
reductions the mask equation implies (Gzip-guided Sparse Attention,
daiwk.github.io, "核心公式"): a wide-window hybrid head is plain causal
attention, a zero-window local head is causal attention inside each block,
and an all-literal sample's literal head is dense causal.  The gradient is
also checked by central finite differences.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as tF

from oracle import attention as A
from oracle import mask as M

LOCAL, LITERAL, HYBRID = M.LOCAL, M.LITERAL, M.HYBRID


def _qkv(T, d, seed, n=3):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(T, d, generator=g, dtype=torch.float64) for _ in range(n)]


def _sdpa(q, k, v, tmask=None, causal=False):
    am = None if tmask is None else torch.from_numpy(tmask)
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        return tF.scaled_dot_product_attention(q[None, None], k[None, None], v[None, None],
                                               attn_mask=am, is_causal=causal)[0, 0]


@pytest.mark.parametrize("cls", [LOCAL, LITERAL, HYBRID])
def test_forward_matches_sdpa(cls):
    b, n, d = 8, 12, 16
    rng = np.random.default_rng(10 + cls)
    fl = (rng.random(n) < 0.45).astype(np.uint8)
    tm = A.dense_token_mask(fl, 1, cls, b)
    q, k, v = _qkv(n * b, d, 20 + cls)
    o_dense, lse_dense = A.forward_dense(q, k, v, tm)
    ref = _sdpa(q, k, v, tm).numpy()
    assert np.abs(o_dense - ref).max() < 1e-12
    s = (q @ k.T / np.sqrt(d)).masked_fill(~torch.from_numpy(tm), -torch.inf)
    assert np.abs(lse_dense - torch.logsumexp(s, dim=1).numpy()).max() < 1e-12
    o_blk, lse_blk = A.forward(q, k, v, M.block_mask(fl, 1, cls), b)
    assert np.abs(o_blk - o_dense).max() < 1e-12
    assert np.abs(lse_blk - lse_dense).max() < 1e-12


def test_wide_window_hybrid_is_causal_attention():
    b, n, d = 4, 16, 8
    fl = (np.random.default_rng(0).random(n) < 0.3).astype(np.uint8)
    q, k, v = _qkv(n * b, d, 1)
    o, _ = A.forward(q, k, v, M.block_mask(fl, n, HYBRID), b)
    assert np.abs(o - _sdpa(q, k, v, causal=True).numpy()).max() < 1e-12


def test_zero_window_local_is_blockwise_causal():
    b, n, d = 8, 6, 8
    fl = np.zeros(n, dtype=np.uint8)
    q, k, v = _qkv(n * b, d, 2)
    o, _ = A.forward(q, k, v, M.block_mask(fl, 0, LOCAL), b)
    for i in range(n):
        r = slice(i * b, (i + 1) * b)
        assert np.abs(o[r] - _sdpa(q[r], k[r], v[r], causal=True).numpy()).max() < 1e-12


def test_all_literal_literal_head_is_causal_attention():
    b, n, d = 4, 10, 8
    fl = np.ones(n, dtype=np.uint8)
    q, k, v = _qkv(n * b, d, 3)
    o, _ = A.forward(q, k, v, M.block_mask(fl, 0, LITERAL), b)
    assert np.abs(o - _sdpa(q, k, v, causal=True).numpy()).max() < 1e-12


@pytest.mark.parametrize("cls", [LOCAL, LITERAL, HYBRID])
def test_backward_matches_autograd(cls):
    b, n, d = 8, 10, 16
    rng = np.random.default_rng(30 + cls)
    fl = (rng.random(n) < 0.5).astype(np.uint8)
    bm = M.block_mask(fl, 2, cls)
    tm = M.token_mask(bm, b)
    q, k, v, do = _qkv(n * b, d, 40 + cls, 4)
    qq, kk, vv = (t.clone().requires_grad_(True) for t in (q, k, v))
    _sdpa(qq, kk, vv, tm).backward(do)
    dq, dk, dv = A.backward_dense(q, k, v, do, tm)
    assert np.abs(dq - qq.grad.numpy()).max() < 1e-11
    assert np.abs(dk - kk.grad.numpy()).max() < 1e-11
    assert np.abs(dv - vv.grad.numpy()).max() < 1e-11
    bq, bk, bv = A.backward(q, k, v, do, bm, b)
    assert np.abs(bq - dq).max() < 1e-11
    assert np.abs(bk - dk).max() < 1e-11
    assert np.abs(bv - dv).max() < 1e-11


def test_backward_finite_differences():
    b, n, d = 4, 6, 4
    fl = np.array([1, 0, 1, 1, 0, 1], dtype=np.uint8)
    bm = M.block_mask(fl, 1, HYBRID)
    q, k, v, do = (t.numpy() for t in _qkv(n * b, d, 50, 4))

    def loss(qx, kx, vx):
        o, _ = A.forward(qx, kx, vx, bm, b)
        return float((o * do).sum())

    dq, dk, dv = A.backward(q, k, v, do, bm, b)
    eps = 1e-6
    rng = np.random.default_rng(0)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            i, j = int(rng.integers(0, n * b)), int(rng.integers(0, d))
            xp, xm = x.copy(), x.copy()
            xp[i, j] += eps
            xm[i, j] -= eps
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - g[i, j]) <= 1e-6 * max(1.0, abs(g[i, j]))


def test_partial_blocks_match_full():
    b, n, d = 8, 9, 8
    fl = (np.random.default_rng(9).random(n) < 0.5).astype(np.uint8)
    bm = M.block_mask(fl, 1, HYBRID)
    q, k, v, do = _qkv(n * b, d, 60, 4)
    o, lse = A.forward(q, k, v, bm, b)
    o2, lse2 = A.forward(q, k, v, bm, b, q_blocks=[2, 7])
    for i in (2, 7):
        r = slice(i * b, (i + 1) * b)
        assert np.array_equal(o[r], o2[r]) and np.array_equal(lse[r], lse2[r])
    dq, dk, dv = A.backward(q, k, v, do, bm, b)
    dq2, dk2, dv2 = A.backward(q, k, v, do, bm, b, q_blocks=[3], k_blocks=[0, 5])
    assert np.abs(dq2[3 * b:4 * b] - dq[3 * b:4 * b]).max() < 1e-13
    for j in (0, 5):
        r = slice(j * b, (j + 1) * b)
        assert np.abs(dk2[r] - dk[r]).max() < 1e-13
        assert np.abs(dv2[r] - dv[r]).max() < 1e-13


def test_batch_wrappers():
    S, H, n, b, d = 2, 4, 6, 4, 8
    rng = np.random.default_rng(11)
    fl = (rng.random((S, n)) < 0.5).astype(np.uint8)
    hc = np.array([LOCAL, LOCAL, LITERAL, HYBRID], dtype=np.uint8)
    g = torch.Generator().manual_seed(5)
    q, k, v, do = (torch.randn(S, H, n * b, d, generator=g, dtype=torch.float64) for _ in range(4))
    o, lse = A.forward_batch(q, k, v, fl, 1, hc, b)
    dq, dk, dv = A.backward_batch(q, k, v, do, fl, 1, hc, b)
    for s in range(S):
        for h in range(H):
            tm = A.dense_token_mask(fl[s], 1, int(hc[h]), b)
            od, ld = A.forward_dense(q[s, h], k[s, h], v[s, h], tm)
            assert np.abs(o[s, h] - od).max() < 1e-12
            gq, gk, gv = A.backward_dense(q[s, h], k[s, h], v[s, h], do[s, h], tm)
            assert np.abs(dq[s, h] - gq).max() < 1e-11
            assert np.abs(dv[s, h] - gv).max() < 1e-11
