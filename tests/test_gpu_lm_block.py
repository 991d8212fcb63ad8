"""gsa_lm_block_fwd / gsa_lm_block_bwd (one ByteLM block around the
block-sparse attention) against the oracle block in float64: the output and
every weight gradient at a small shape (two samples of 17 blocks, so the
attention's 128-row tiles end ragged), the output on sampled query blocks at
the full 8x8K, D = 768 shape, repeatability of the backward, and a fixed
(BigBird) mask through the same calls."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import deflate1
from oracle import flags as ofl
from oracle import lm_block as olm
from oracle import mask as om

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gsa():
    from content_adaptive_block_b200 import build
    build.build()
    import content_adaptive_block_b200 as g
    return g


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _classes(H):
    return [0] * (H // 2) + [1] * (H // 4) + [2] * (H - H // 2 - H // 4)


def _gzip_masks(x, b, w, classes):
    fl = ofl.literal_flags(deflate1.block_lengths(x, b), b)
    bm = [[om.block_mask(fl[s], w, c) for c in classes] for s in range(x.shape[0])]
    return bm, [[torch.from_numpy(om.token_mask(m, b)) for m in row] for row in bm]


def _small_case(gsa, seed, fixed=None):
    c = W.LM_BLOCK_SMALL
    S, L, D, H, F, w = c["S"], c["L"], c["D"], c["H"], c["F"], c["w"]
    classes = _classes(H)
    x = W.custom_bytes(S, L, ("uniform", 0.2, 0.6), seed=seed, salt=31)
    wt = W.lm_weights(D, F, seed=seed, device="cuda")
    xd = torch.from_numpy(x).cuda()
    if fixed is None:
        _, _, csr = gsa.gsa_mask_pipeline(xd, 64, w)
        bm, tm = _gzip_masks(x, 64, w, classes)
    else:
        rnd = W.random_words(S, L // 64, fixed["r"], seed=seed)
        csr = gsa.gsa_build_fixed_csr(fixed["kind"], S, L // 64, fixed["w"], fixed["g"],
                                      torch.from_numpy(rnd.view(np.int32)).cuda())
        bm = [[om.fixed_block_mask(fixed["kind"], L // 64, fixed["w"], fixed["g"], rnd[s])] * H for s in range(S)]
        tm = [[torch.from_numpy(om.token_mask(m, 64)) for m in row] for row in bm]
    g = torch.Generator(device="cpu")
    g.manual_seed(seed + 5)
    dy = torch.randn((S, L, D), generator=g).bfloat16().cuda()
    return x, xd, wt, csr, classes, tm, dy, H


@pytest.mark.parametrize("fixed", [None, W.FIXED_MASKS["bigbird"]], ids=["gzip", "bigbird"])
def test_block_matches_oracle(gsa, fixed):
    x, xd, wt, csr, classes, tm, dy, H = _small_case(gsa, 1, fixed)
    y, ws = gsa.gsa_lm_block_fwd(xd, wt, csr, classes)
    grads = gsa.gsa_lm_block_bwd(xd, wt, csr, classes, dy, ws)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    w64 = {k: v.double().cpu().numpy() for k, v in wt.items()}
    y_ref, g_ref = olm.block_forward_backward(x, w64, tm, H, dy.double().cpu().numpy())
    assert _rel(y.double().cpu().numpy(), y_ref) <= 1e-2
    for n in gsa.LM_WEIGHTS:
        got = grads[n].double().cpu().numpy()
        if n == "emb":   # rows of bytes that occur; the rest must be exactly zero
            used = np.zeros(256, dtype=bool)
            used[np.unique(x)] = True
            assert np.all(got[~used] == 0.0)
            got, want = got[used], g_ref[n][used]
        else:
            want = g_ref[n]
        assert _rel(got, want) <= 2e-2, n


def test_backward_is_repeatable(gsa):
    x, xd, wt, csr, classes, tm, dy, H = _small_case(gsa, 2)
    y, ws = gsa.gsa_lm_block_fwd(xd, wt, csr, classes)
    g1 = {k: v.clone() for k, v in gsa.gsa_lm_block_bwd(xd, wt, csr, classes, dy, ws).items()}
    y2, ws = gsa.gsa_lm_block_fwd(xd, wt, csr, classes, workspace=ws)
    g2 = gsa.gsa_lm_block_bwd(xd, wt, csr, classes, dy, ws)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    for n in gsa.LM_WEIGHTS:
        assert torch.equal(g1[n], g2[n]), n


def test_full_size_forward_on_sampled_blocks(gsa):
    wl = W.WORKLOADS["b8_8k"]
    c = W.LM_BLOCK
    D, H, F = c["D"], c["H"], c["F"]
    classes = [int(v) for v in wl.head_classes()]
    x = W.batch_bytes(wl, seed=0)
    xd = torch.from_numpy(x).cuda()
    wt = W.lm_weights(D, F, seed=3, device="cuda")
    _, _, csr = gsa.gsa_mask_pipeline(xd, wl.b, wl.w)
    y, _ = gsa.gsa_lm_block_fwd(xd, wt, csr, classes)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    w64 = {k: v.double().cpu().numpy() for k, v in wt.items()}
    fl = ofl.literal_flags(deflate1.block_lengths(x[[0, wl.S - 1]], wl.b), wl.b)
    yc = y.double().cpu().numpy()
    for i, s in enumerate((0, wl.S - 1)):
        bm = [om.block_mask(fl[i], wl.w, cl) for cl in classes]
        rows, ref = olm.block_rows_forward(x[s], w64, bm, H, wl.b, [0, 5, wl.N // 2, wl.N - 1])
        assert _rel(yc[s, rows], ref) <= 1e-2, s
