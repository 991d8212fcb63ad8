"""gsa_build_fixed_csr (Longformer, BigBird block masks) against the oracle's
fixed masks: every list and both orders bit for bit, then the attention
forward and backward through those lists against the oracle attention on the
same mask (sampled query / key blocks at the 8x8K shape)."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as oatt
from oracle import mask as om

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gsa():
    from content_adaptive_block_b200 import build
    build.build()
    import content_adaptive_block_b200 as g
    return g


def _build(gsa, kind, B, n, w, g, r, seed=0):
    rnd = W.random_words(B, n, r, seed) if kind == om.BIGBIRD else None
    t = torch.from_numpy(rnd.view(np.int32)).cuda() if rnd is not None else None
    csr = gsa.gsa_build_fixed_csr(kind, B, n, w, g, t, device="cuda")
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    return csr, rnd


def _check(gsa, kind, B, n, w, g, r, seed=0):
    csr, rnd = _build(gsa, kind, B, n, w, g, r, seed)
    qo, ko = csr.q_order.cpu().numpy(), csr.k_order.cpu().numpy()
    for s in range(B):
        m = om.fixed_block_mask(kind, n, w, g, rnd[s] if rnd is not None else None)
        want_r = [list(x) for x in om.row_lists(m)]
        want_c = [list(x) for x in om.col_lists(m)]
        for c in range(3):
            assert csr.rows(s, c) == want_r, (s, c)
            assert csr.cols(s, c) == want_c, (s, c)
            assert qo[s, c].tolist() == list(range(n - 1, -1, -1))
            assert ko[s, c].tolist() == list(range(n))
        assert int(csr.row_ptr[s, 0, -1]) == om.live_pairs(m)
    return csr, rnd


@pytest.mark.parametrize("n", [1, 2, 31, 32, 33, 128, 1000])
@pytest.mark.parametrize("w,g", [(0, 0), (1, 2), (4, 1), (3, 40)])
def test_longformer_lists(gsa, n, w, g):
    _check(gsa, om.LONGFORMER, 2, n, w, g, 0)


@pytest.mark.parametrize("n", [1, 2, 33, 128, 1000])
@pytest.mark.parametrize("w,g,r", [(1, 2, 3), (0, 0, 1), (2, 0, 8), (0, 5, 8)])
def test_bigbird_lists(gsa, n, w, g, r):
    _check(gsa, om.BIGBIRD, 3, n, w, g, r, seed=n + r)


def test_largest_lists(gsa):
    # the largest mask the call takes, with the most random blocks: sampled rows and columns
    n, w, g, r = 8192, 2, 3, 8
    csr, rnd = _build(gsa, om.BIGBIRD, 1, n, w, g, r, seed=5)
    m = om.fixed_block_mask(om.BIGBIRD, n, w, g, rnd[0])
    rp, cp = csr.row_ptr[0, 2].cpu().numpy(), csr.col_ptr[0, 2].cpu().numpy()
    ci, ri = csr.col_idx[0, 2].cpu().numpy(), csr.row_idx[0, 2].cpu().numpy()
    assert rp[-1] == cp[-1] == m.sum()
    for i in (0, 1, 2, 3, 4, 5, 4095, 8190, 8191):
        assert ci[rp[i]:rp[i + 1]].tolist() == np.nonzero(m[i])[0].tolist(), i
        assert ri[cp[i]:cp[i + 1]].tolist() == np.nonzero(m[:, i])[0].tolist(), i


def test_longformer_without_globals_matches_the_local_class(gsa):
    # the adaptive builder's local class is the same sliding window
    B, n, w = 2, 96, 3
    fl = torch.zeros((B, n), dtype=torch.uint8, device="cuda")
    ref = gsa.gsa_build_block_csr(fl, w)
    csr, _ = _build(gsa, om.LONGFORMER, B, n, w, 0, 0)
    for s in range(B):
        assert csr.rows(s, 1) == ref.rows(s, 0)
        assert csr.cols(s, 2) == ref.cols(s, 0)


@pytest.mark.parametrize("name", list(W.FIXED_MASKS))
def test_attention_on_fixed_masks(gsa, name):
    cfg = W.FIXED_MASKS[name]
    wl = W.WORKLOADS["b8_8k"]
    n = wl.N
    csr, rnd = _build(gsa, cfg["kind"], wl.S, n, cfg["w"], cfg["g"], cfg["r"], seed=11)
    hc = [int(c) for c in wl.head_classes()]
    q, k, v, do = W.qkv(wl, seed=3, device="cuda", grad=True)
    o, lse = gsa.gsa_attn_fwd(q, k, v, csr, hc, wl.b)
    dq, dk, dv = gsa.gsa_attn_bwd(q, k, v, o, lse, do, csr, hc, wl.b)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    qs, ks, vs, dos = (x.float().cpu().numpy() for x in (q, k, v, do))
    got = [x.float().cpu().numpy() for x in (o, lse, dq, dk, dv)]
    rng = np.random.default_rng(7)
    for s, h in ((0, 0), (wl.S - 1, wl.H - 1), (3, 7)):
        m = om.fixed_block_mask(cfg["kind"], n, cfg["w"], cfg["g"], rnd[s] if rnd is not None else None)
        qb = sorted(set([0, 1, n - 1] + rng.integers(0, n, 3).tolist()))
        kb = sorted(set([0, n - 1] + rng.integers(0, n, 2).tolist()))
        o_ref, lse_ref = oatt.forward(qs[s, h], ks[s, h], vs[s, h], m, wl.b, q_blocks=qb)
        dq_ref, dk_ref, dv_ref = oatt.backward(qs[s, h], ks[s, h], vs[s, h], dos[s, h], m, wl.b,
                                               q_blocks=qb, k_blocks=kb)
        rows = np.concatenate([np.arange(i * wl.b, (i + 1) * wl.b) for i in qb])
        keys = np.concatenate([np.arange(j * wl.b, (j + 1) * wl.b) for j in kb])
        assert np.abs(got[0][s, h, rows] - o_ref[rows]).max() <= 2e-2
        assert np.abs(got[1][s, h, rows] - lse_ref[rows]).max() <= 1e-3   # LSE bar of every bf16 test
        for g_, r_, idx in ((got[2], dq_ref, rows), (got[3], dk_ref, keys), (got[4], dv_ref, keys)):
            err = np.linalg.norm(g_[s, h, idx] - r_[idx]) / np.linalg.norm(r_[idx])
            assert err <= 2e-2, (name, s, h, err)
