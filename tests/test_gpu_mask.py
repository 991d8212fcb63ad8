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
