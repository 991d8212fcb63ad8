"""gsa_mask_pipeline (lengths -> flags -> block lists in one launch) against
the three separate calls, which test_gpu_mask.py pins to the oracle, and its
lengths against the oracle directly: every output must match bit for bit.
Cases cover CTAs that straddle samples (blocks per sample not a multiple of
four), one block per sample, the largest supported list (1024 blocks), the
mask-sweep batches at full size, two calls in a row on one counter
(each call leaves it zero), subsets of the head classes, and attention on
the pipeline's lists (the local class implicit: not stored, derived by the
attention kernels)."""
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


def _lists(csr, s, c):
    """Pointers, pairing orders and entries of (sample s, class c)."""
    rp, cp = csr.row_ptr[s, c].cpu().numpy(), csr.col_ptr[s, c].cpu().numpy()
    return (rp, cp, csr.q_order[s, c].cpu().numpy(), csr.k_order[s, c].cpu().numpy(),
            csr.col_idx[s, c, :rp[-1]].cpu().numpy(), csr.row_idx[s, c, :cp[-1]].cpu().numpy())


def _same(gsa, x: np.ndarray, b: int, w: int, counters=None, head_classes=None):
    """The pipeline against the three calls: lengths and flags bit for bit, and
    every (sample, class) list of the classes in use equal to the three calls'
    (the local class is implicit: marked, not stored)."""
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    ln_ref = gsa.gsa_block_lengths(t, b)
    fl_ref = gsa.gsa_literal_flags(ln_ref)
    csr_ref = gsa.gsa_build_block_csr(fl_ref, w)
    ln, fl, csr = gsa.gsa_mask_pipeline(t, b, w, counters=counters, head_classes=head_classes)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    assert torch.equal(ln, ln_ref)
    assert torch.equal(fl, fl_ref)
    assert csr.w == csr_ref.w == w
    used = {0, 1, 2} if head_classes is None else set(head_classes)
    assert csr.classes == sum(1 << c for c in used) | (8 if 0 in used else 0)
    assert not csr.stored(0) if 0 in used else True
    for s in range(x.shape[0]):
        for c in sorted(used - {0}):
            for got, want in zip(_lists(csr, s, c), _lists(csr_ref, s, c)):
                assert np.array_equal(got, want), (s, c)
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


@pytest.mark.parametrize("B,nblk,b,w", [(1024, 32, 64, 2), (2048, 16, 128, 1), (1024, 16, 16, 1)])
def test_pipeline_list_jobs_per_warp(gsa, B, nblk, b, w):
    """Many samples of short lists: more list jobs than CTAs, so each warp
    takes jobs of its own (the warp-job path of phase 2)."""
    x = W.custom_bytes(B, nblk * b, ("uniform", 0.2, 0.6), seed=B + nblk)
    ln = _same(gsa, x, b, w)
    assert np.array_equal(ln, deflate1.block_lengths(x, b, nthreads=8))


def test_pipeline_narrow_ctas_small_blocks(gsa):
    """Blocks of at most 32 bytes, more list jobs than SMs and short lists:
    the narrow CTA shape of the smallest block size, one job per CTA."""
    x = W.custom_bytes(256, 64 * 32, ("uniform", 0.2, 0.6), seed=31)
    ln = _same(gsa, x, 32, 2)
    assert np.array_equal(ln, deflate1.block_lengths(x, 32, nthreads=8))


def test_pipeline_reuses_its_counters(gsa):
    wl = W.WORKLOADS["b8_4k"]
    counters = torch.zeros(1, dtype=torch.int32, device="cuda")
    for seed in (0, 1, 2):
        _same(gsa, W.batch_bytes(wl, seed=seed), wl.b, wl.w, counters=counters)
        assert int(counters.abs().sum().item()) == 0


@pytest.mark.parametrize("head_classes", [[0], [1, 2], [2, 0, 0], [1]])
def test_pipeline_classes_in_use(gsa, head_classes):
    wl = W.WORKLOADS["b8_4k"]
    _same(gsa, W.batch_bytes(wl, seed=4), wl.b, wl.w, head_classes=head_classes)


def test_attention_on_pipeline_lists(gsa):
    """Forward and backward on the pipeline's lists (the local class implicit)
    give the three-call lists' results bit for bit, at d = 64 and d = 128, and
    the float32 forward likewise."""
    wl = W.WORKLOADS["b8_4k"]
    hc = [int(c) for c in wl.head_classes()]
    t = torch.from_numpy(W.batch_bytes(wl, seed=5)).cuda()
    csr_ref = gsa.gsa_build_block_csr(gsa.gsa_literal_flags(gsa.gsa_block_lengths(t, wl.b)), wl.w)
    _, _, csr = gsa.gsa_mask_pipeline(t, wl.b, wl.w)
    for d in (64, 128):
        q, k, v, do = (x.cuda() for x in W.random_tensors((wl.S, wl.H, wl.L, d), 4, torch.bfloat16, seed=d))
        outs = []
        for c in (csr_ref, csr):
            o, lse = gsa.gsa_attn_fwd(q, k, v, c, hc, wl.b)
            outs.append([o, lse, *gsa.gsa_attn_bwd(q, k, v, o, lse, do, c, hc, wl.b)])
        torch.cuda.synchronize()
        assert gsa.gsa_device_error() == 0
        for a, b_ in zip(*outs):
            assert torch.equal(a, b_), d

    # the float32 path (CUDA cores) on the tiny workload
    wl = W.WORKLOADS["tiny_fp32"]
    hc = [int(c) for c in wl.head_classes()]
    t = torch.from_numpy(W.batch_bytes(wl, seed=6)).cuda()
    csr_ref = gsa.gsa_build_block_csr(gsa.gsa_literal_flags(gsa.gsa_block_lengths(t, wl.b)), wl.w)
    _, _, csr = gsa.gsa_mask_pipeline(t, wl.b, wl.w)
    q, k, v = (x.cuda() for x in W.random_tensors((wl.S, wl.H, wl.L, wl.d), 3, torch.float32, seed=7))
    o_ref, lse_ref = gsa.gsa_attn_fwd(q, k, v, csr_ref, hc, wl.b)
    o, lse = gsa.gsa_attn_fwd(q, k, v, csr, hc, wl.b)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


@pytest.mark.parametrize("B,nblk,w", [(2, 17, 0), (2, 9, 20), (1, 33, 3), (3, 1, 2)])
@pytest.mark.parametrize("d", [64, 128])
def test_implicit_local_window_edges(gsa, B, nblk, w, d):
    """The implicit local window at its edges (w = 0, w past the first block,
    odd block counts, one block) against the stored lists of the three calls:
    forward and backward bit for bit, local heads only and mixed."""
    b = 64
    x = W.custom_bytes(B, nblk * b, ("uniform", 0.2, 0.6), seed=nblk * 10 + w)
    t = torch.from_numpy(x).cuda()
    csr_ref = gsa.gsa_build_block_csr(gsa.gsa_literal_flags(gsa.gsa_block_lengths(t, b)), w)
    for hc in ([0, 0], [0, 1, 2, 0]):
        _, _, csr = gsa.gsa_mask_pipeline(t, b, w, head_classes=hc)
        q, k, v, do = (y.cuda() for y in W.random_tensors((B, len(hc), nblk * b, d), 4, torch.bfloat16, seed=d + w))
        outs = []
        for c in (csr_ref, csr):
            o, lse = gsa.gsa_attn_fwd(q, k, v, c, hc, b)
            outs.append([o, lse, *gsa.gsa_attn_bwd(q, k, v, o, lse, do, c, hc, b)])
        torch.cuda.synchronize()
        assert gsa.gsa_device_error() == 0
        for a, b_ in zip(*outs):
            assert torch.equal(a, b_), (hc, d)
