"""GPU parity of the mask stage against the oracle: gzip lengths, literal
flags and the per-class block lists must match bit for bit."""
import os
import random

import numpy as np
import pytest
import torch

import workloads as W
from oracle import deflate1, flags as oflags, mask as omask

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def gsa():
    from content_adaptive_block_b200 import build
    build.build()
    import content_adaptive_block_b200 as g
    return g


def _gpu_lengths(gsa, x: np.ndarray, b: int) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    out = gsa.gsa_block_lengths(t, b)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_lengths_workloads(gsa, name):
    wl = W.WORKLOADS[name]
    x = W.batch_bytes(wl, seed=0)
    assert np.array_equal(_gpu_lengths(gsa, x, wl.b), deflate1.block_lengths(x, wl.b, nthreads=8))


@pytest.mark.parametrize("b,f", W.MASK_SWEEP)
def test_lengths_mask_sweep_full_size(gsa, b, f):
    # 256 samples x 8192 bytes: every block of the full launch is checked
    wl = W.mask_sweep(b, f)
    x = W.batch_bytes(wl, seed=1)
    got = _gpu_lengths(gsa, x, b)
    want = deflate1.block_lengths(x, b, nthreads=os.cpu_count() or 8)
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} mismatches, first {bad[:3].tolist()}"


def _families(rnd, b):
    words = [bytes(rnd.choice(b"abcdefghijklmnopqrstuvwxyz") for _ in range(rnd.randint(2, 5))) for _ in range(16)]
    ph = b" ".join(rnd.choice(words) for _ in range(rnd.randint(1, 3))) + b" "
    out = [
        bytes(rnd.getrandbits(8) for _ in range(b)),
        bytes(rnd.randint(32, 126) for _ in range(b)),
        (ph * (b // len(ph) + 2))[:b],
        bytes([rnd.randrange(256)]) * b,
        bytes(rnd.randint(0, 3) for _ in range(b)),
        bytes(rnd.randint(97, 98) for _ in range(b)),
    ]
    x = bytearray(rnd.randint(97, 100) for _ in range(b))
    z = rnd.randint(0, b)
    x[z:] = bytes(b - z)
    out.append(bytes(x))
    head = bytes(rnd.randint(97, 99) for _ in range(rnd.randint(3, 6)))
    out.append((head * (b // len(head) + 1))[:b])
    return out


@pytest.mark.parametrize("b", [1, 2, 3, 4, 5, 7, 8, 16, 31, 32, 33, 64, 100, 127, 128])
def test_lengths_block_families(gsa, b):
    rnd = random.Random(77 + b)
    blocks = []
    for _ in range(max(64, 4096 // b)):
        blocks.extend(_families(rnd, b))
    x = np.frombuffer(b"".join(blocks), dtype=np.uint8).reshape(len(blocks), b)
    got = _gpu_lengths(gsa, x, b)
    want = deflate1.block_lengths(x, b, nthreads=8)
    bad = np.argwhere(got != want)
    assert bad.size == 0, [(int(i), bytes(x[i]).hex(), int(got[i, 0]), int(want[i, 0])) for i, _ in bad[:3]]


def test_lengths_code_length_overflow_fixtures(gsa):
    rows = []
    for line in open(os.path.join(HERE, "golden", "code_length_overflow.txt")):
        if line.startswith("#") or not line.strip():
            continue
        b, _, hx = line.split()
        if int(b) <= 128:
            rows.append(bytes.fromhex(hx))
    assert rows
    x = np.frombuffer(b"".join(rows), dtype=np.uint8).reshape(len(rows), 128)
    assert np.array_equal(_gpu_lengths(gsa, x, 128), deflate1.block_lengths(x, 128))


@pytest.mark.parametrize("S,b", [(23, 64), (39, 64), (95, 64), (7, 128), (47, 128), (161, 32)])
def test_lengths_blocks_per_warp(gsa, S, b):
    """Batch sizes whose blocks fill one wave of resident warps at 2, 4, 8 or
    16 blocks a warp (the launcher picks the fewest that fit), so every
    chunk size of the lengths kernel runs, with a ragged last chunk."""
    x = W.custom_bytes(S, 8192 - b, ("uniform", 0.2, 0.6), seed=S * 7 + b)
    assert np.array_equal(_gpu_lengths(gsa, x, b), deflate1.block_lengths(x, b, nthreads=8))


def test_lengths_several_blocks_per_sample(gsa):
    x = W.custom_bytes(3, 64 * 37, ("fixed", 0.4), seed=5)[:, : 64 * 37]
    for b in (16, 32, 64):
        L = (x.shape[1] // b) * b
        xx = np.ascontiguousarray(x[:, :L])
        assert np.array_equal(_gpu_lengths(gsa, xx, b), deflate1.block_lengths(xx, b))


def test_flags_match_oracle(gsa):
    rng = np.random.default_rng(3)
    for n in (1, 2, 3, 16, 64, 128, 1024, 1500):
        ln = rng.integers(20, 90, size=(5, n)).astype(np.int32)
        ln[1] = 40                     # all equal: no literal block
        ln[2, : n // 2] = 30
        ln[2, n // 2:] = 31
        got = gsa.gsa_literal_flags(torch.from_numpy(ln).cuda()).cpu().numpy()
        assert np.array_equal(got, oflags.literal_flags(ln, 64))


def _check_lists(gsa, fl: np.ndarray, w: int):
    csr = gsa.gsa_build_block_csr(torch.from_numpy(fl.astype(np.uint8)).cuda(), w)
    torch.cuda.synchronize()
    B, n = fl.shape
    qo = csr.q_order.cpu().numpy()
    ko = csr.k_order.cpu().numpy()
    for s in range(B):
        for c in (0, 1, 2):
            m = omask.block_mask(fl[s], w, c)
            rows = csr.rows(s, c)
            cols = csr.cols(s, c)
            assert [list(r) for r in omask.row_lists(m)] == rows, (s, c)
            assert [list(x) for x in omask.col_lists(m)] == cols, (s, c)
            assert sorted(qo[s, c].tolist()) == list(range(n))
            assert sorted(ko[s, c].tolist()) == list(range(n))
            if c != 0:
                lit = np.nonzero(fl[s])[0]
                nl = len(lit)
                assert qo[s, c, :nl].tolist() == lit[::-1].tolist()
                assert ko[s, c, :nl].tolist() == lit.tolist()


@pytest.mark.parametrize("n", [1, 2, 3, 5, 16, 63, 64, 128, 1024])
def test_block_lists_match_mask(gsa, n):
    rng = np.random.default_rng(n)
    fl = (rng.random((3, n)) < rng.random((3, 1))).astype(np.uint8)
    for w in sorted({0, 1, 2, 4, max(0, n - 1), n + 3}):
        _check_lists(gsa, fl, w)


def test_block_lists_special_flags(gsa):
    n = 40
    fl = np.stack([np.ones(n), np.zeros(n), np.eye(1, n, n - 1)[0]]).astype(np.uint8)
    _check_lists(gsa, fl, 2)


def test_pipeline_end_to_end_mask(gsa):
    wl = W.WORKLOADS["b8_8k"]
    x = W.batch_bytes(wl, seed=2)
    ln = gsa.gsa_block_lengths(torch.from_numpy(x).cuda(), wl.b)
    fl = gsa.gsa_literal_flags(ln)
    csr = gsa.gsa_build_block_csr(fl, wl.w)
    want_fl = oflags.literal_flags(deflate1.block_lengths(x, wl.b), wl.b)
    assert np.array_equal(fl.cpu().numpy(), want_fl)
    for s in range(wl.S):
        for c in (0, 1, 2):
            assert csr.rows(s, c) == [list(r) for r in omask.row_lists(omask.block_mask(want_fl[s], wl.w, c))]


@pytest.mark.parametrize("head_classes", [[0, 0], [1], [2, 2, 1], [1, 0, 2]])
def test_block_lists_for_the_classes_in_use(gsa, head_classes):
    """gsa_build_block_csr with head classes builds the lists of exactly the
    classes that appear (the other classes' slots keep what they held) and
    records them; attention on those heads matches the all-class build bit
    for bit, and a head of a class not built is refused."""
    B, n, w, b, d = 2, 33, 2, 64, 64
    rng = np.random.default_rng(len(head_classes))
    fl = torch.from_numpy((rng.random((B, n)) < 0.4).astype(np.uint8)).cuda()
    full = gsa.gsa_build_block_csr(fl, w)
    part = gsa.BlockCsr(B, n, fl.device)
    for t in (part.row_ptr, part.col_ptr, part.q_order, part.k_order, part.col_idx, part.row_idx):
        t.fill_(-7)
    gsa.gsa_build_block_csr(fl, w, part, head_classes=head_classes)
    torch.cuda.synchronize()
    want = sum(1 << c for c in set(head_classes))
    assert part.classes == want and full.classes == 7
    for c in range(3):
        if (want >> c) & 1:
            for s in range(B):
                assert part.rows(s, c) == full.rows(s, c) and part.cols(s, c) == full.cols(s, c)
            assert torch.equal(part.q_order[:, c], full.q_order[:, c])
            assert torch.equal(part.k_order[:, c], full.k_order[:, c])
        else:
            assert (part.row_ptr[:, c] == -7).all() and (part.q_order[:, c] == -7).all()
    H = len(head_classes)
    q, k, v = (t.cuda() for t in W.random_tensors((B, H, n * b, d), 3, torch.bfloat16, seed=40 + H))
    o1, l1 = gsa.gsa_attn_fwd(q, k, v, full, head_classes, b)
    o2, l2 = gsa.gsa_attn_fwd(q, k, v, part, head_classes, b)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    missing = [c for c in range(3) if not (want >> c) & 1]
    if missing:
        with pytest.raises(RuntimeError):
            gsa.gsa_attn_fwd(q, k, v, part, [missing[0]] * H, b)
