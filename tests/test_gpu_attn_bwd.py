"""GPU parity of the attention backward against the float64 oracle.

Bar: relative L2 error <= 2e-2 for each of dQ, dK, dV per (sample, head),
over the rows compared.  The GPU backward takes the GPU forward's O and LSE,
as in training; the oracle recomputes everything in float64 from the same
bf16-rounded Q, K, V and dO."""
import numpy as np
import pytest
import torch

import workloads as W
from parity_sampling import class_pairs
from oracle import attention as oatt, deflate1, flags as oflags, mask as omask

pytestmark = pytest.mark.gpu

TOL_REL_L2 = 2e-2


@pytest.fixture(scope="module")
def gsa():
    from content_adaptive_block_b200 import build
    build.build()
    import content_adaptive_block_b200 as g
    return g


def _run(gsa, q, k, v, do, fl, w, hc, b):
    csr = gsa.gsa_build_block_csr(torch.from_numpy(fl.astype(np.uint8)).cuda(), w)
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = gsa.gsa_attn_fwd(qc, kc, vc, csr, list(hc), b)
    dq, dk, dv = gsa.gsa_attn_bwd(qc, kc, vc, o, lse, dc, csr, list(hc), b)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    return [t.float().cpu().numpy() for t in (dq, dk, dv)]


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _compare(got, q, k, v, do, fl, w, hc, b, pairs=None, q_blocks=None, k_blocks=None):
    S, H = q.shape[:2]
    worst = 0.0
    for s in range(S):
        for h in range(H):
            if pairs is not None and (s, h) not in pairs:
                continue
            m = omask.block_mask(fl[s], w, int(hc[h]))
            ref = oatt.backward(q[s, h].float(), k[s, h].float(), v[s, h].float(), do[s, h].float(), m, b,
                                q_blocks=q_blocks, k_blocks=k_blocks)
            for name, g, r in zip(("dq", "dk", "dv"), got, ref):
                sel = ~np.isnan(r[:, 0])
                e = _rel(g[s, h][sel], r[sel])
                worst = max(worst, e)
                assert e <= TOL_REL_L2, (name, s, h, e)
    return worst


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n,w", [(1, 1), (2, 0), (3, 1), (9, 2), (16, 2), (33, 4)])
def test_bwd_small_shapes(gsa, d, n, w):
    S, H, b = 2, 4, 64
    rng = np.random.default_rng(n * 7 + w + d)
    fl = (rng.random((S, n)) < 0.45).astype(np.uint8)
    hc = np.array([0, 1, 2, 2], dtype=np.uint8)
    q, k, v, do = W.random_tensors((S, H, n * b, d), 4, torch.bfloat16, seed=100 + n + d)
    got = _run(gsa, q, k, v, do, fl, w, hc, b)
    _compare(got, q, k, v, do, fl, w, hc, b)


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_special_masks(gsa, d):
    S, H, n, b = 3, 3, 12, 64
    fl = np.stack([np.ones(n), np.zeros(n), (np.arange(n) % 3 == 0)]).astype(np.uint8)
    hc = np.array([0, 1, 2], dtype=np.uint8)
    q, k, v, do = W.random_tensors((S, H, n * b, d), 4, torch.bfloat16, seed=9 + d)
    for w in (0, 2, n):
        got = _run(gsa, q, k, v, do, fl, w, hc, b)
        _compare(got, q, k, v, do, fl, w, hc, b)


def test_bwd_b8_8k_sampled(gsa):
    wl = W.WORKLOADS["b8_8k"]
    x = W.batch_bytes(wl)
    fl = oflags.literal_flags(deflate1.block_lengths(x, wl.b, 8), wl.b)
    q, k, v, do = W.qkv(wl, seed=0, grad=True)
    got = _run(gsa, q, k, v, do, fl, wl.w, wl.head_classes(), wl.b)
    hc = wl.head_classes()
    rng = np.random.default_rng(5)
    pairs = class_pairs(wl.S, hc, 4, seed=5)   # 4 distinct (sample, head) per class
    assert len(pairs) == 12
    blocks = sorted(set([0, 1, wl.N - 1] + rng.integers(0, wl.N, 10).tolist()))
    _compare(got, q, k, v, do, fl, wl.w, hc, wl.b, pairs=pairs, q_blocks=blocks, k_blocks=blocks)


def test_bwd_b1_64k_sampled(gsa):
    wl = W.WORKLOADS["b1_64k"]
    x = W.batch_bytes(wl)
    fl = oflags.literal_flags(deflate1.block_lengths(x, wl.b, 8), wl.b)
    q, k, v, do = W.qkv(wl, seed=0, grad=True)
    got = _run(gsa, q, k, v, do, fl, wl.w, wl.head_classes(), wl.b)
    hc = wl.head_classes()
    lit = np.nonzero(fl[0])[0]
    blocks = sorted(set([0, 1, wl.N - 1, int(lit[0]), int(lit[-1]), int(lit[len(lit) // 2])] +
                        np.random.default_rng(2).integers(0, wl.N, 8).tolist()))
    pairs = class_pairs(wl.S, hc, 4, seed=2)   # 4 distinct heads per class (the one sample)
    assert len(pairs) == 12
    _compare(got, q, k, v, do, fl, wl.w, hc, wl.b, pairs=pairs, q_blocks=blocks, k_blocks=blocks)
