"""gsa_mask_pipeline (lengths -> flags -> block lists in one launch) against
the three separate calls, which test_gpu_mask.py pins to the oracle, and its
lengths against the oracle directly: every output must match bit for bit.
Cases cover CTAs that straddle samples (blocks per sample not a multiple of
four), one block per sample, the largest supported list (1024 blocks), the
mask-sweep batches at full size, and two calls in a row on one counter
buffer (each call leaves it zero)."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import deflate1

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gsa():
    from content_adaptive_block_b200 import build
    build.build()
    import content_adaptive_block_b200 as g
    return g


def _lists(csr):
    """(row_ptr, col_ptr, q_order, k_order, per-(sample, class) entries) on the host."""
    rp, cp = csr.row_ptr.cpu().numpy(), csr.col_ptr.cpu().numpy()
    ci, ri = csr.col_idx.cpu().numpy(), csr.row_idx.cpu().numpy()
    ents = []
    for s in range(rp.shape[0]):
        for c in range(3):
            ents.append((ci[s, c, :rp[s, c, -1]].copy(), ri[s, c, :cp[s, c, -1]].copy()))
    return rp, cp, csr.q_order.cpu().numpy(), csr.k_order.cpu().numpy(), ents


def _same(gsa, x: np.ndarray, b: int, w: int, counters=None):
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    ln_ref = gsa.gsa_block_lengths(t, b)
    fl_ref = gsa.gsa_literal_flags(ln_ref)
    csr_ref = gsa.gsa_build_block_csr(fl_ref, w)
    ln, fl, csr = gsa.gsa_mask_pipeline(t, b, w, counters=counters)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    assert torch.equal(ln, ln_ref)
    assert torch.equal(fl, fl_ref)
    assert csr.w == csr_ref.w == w
    a, r = _lists(csr), _lists(csr_ref)
    for got, want in zip(a[:4], r[:4]):
        assert np.array_equal(got, want)
    for (gc, gr), (wc, wr) in zip(a[4], r[4]):
        assert np.array_equal(gc, wc) and np.array_equal(gr, wr)
    return ln.cpu().numpy()


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_pipeline_workloads(gsa, name):
    wl = W.WORKLOADS[name]
    x = W.batch_bytes(wl, seed=0)
    ln = _same(gsa, x, wl.b, wl.w)
    assert np.array_equal(ln, deflate1.block_lengths(x, wl.b, nthreads=8))


@pytest.mark.parametrize("b", [32, 64, 128])
def test_pipeline_mask_sweep_full_size(gsa, b):
    wl = W.mask_sweep(b, 0.3)
    _same(gsa, W.batch_bytes(wl, seed=1), b, wl.w)


@pytest.mark.parametrize("B,nblk,b,w", [(3, 5, 32, 1), (7, 1, 64, 2), (5, 6, 16, 0), (2, 1024, 16, 3),
                                         (9, 13, 128, 4)])
def test_pipeline_odd_shapes(gsa, B, nblk, b, w):
    x = W.custom_bytes(B, nblk * b, ("uniform", 0.2, 0.6), seed=B * 100 + nblk)
    ln = _same(gsa, x, b, w)
    assert np.array_equal(ln, deflate1.block_lengths(x, b, nthreads=8))


def test_pipeline_reuses_its_counters(gsa):
    wl = W.WORKLOADS["b8_4k"]
    counters = torch.zeros(wl.S, dtype=torch.int32, device="cuda")
    for seed in (0, 1, 2):
        _same(gsa, W.batch_bytes(wl, seed=seed), wl.b, wl.w, counters=counters)
        assert int(counters.abs().sum().item()) == 0
