"""Pins for the oracle's gzip level-1 length (CPU only).

What "gzip level 1" means is fixed outside the oracle: the host zlib
library (classic zlib, the library Python's gzip module calls) produces the
stream the method measures.  The oracle is checked against it byte for byte,
by inflating its output back, and on a few streams whose size follows by hand
from the RFC 1951 code tables.
"""
import gzip
import os
import random
import zlib

import numpy as np
import pytest

from oracle import deflate1

HERE = os.path.dirname(os.path.abspath(__file__))


def _zraw(x: bytes) -> bytes:
    return zlib.compress(x, 1, -15)


def test_host_zlib_is_classic():
    # zlib-ng's level 1 uses a different match finder; the pins assume zlib.
    assert "ng" not in zlib.ZLIB_RUNTIME_VERSION.lower()
    assert zlib.ZLIB_RUNTIME_VERSION.startswith("1.")


# Sizes derived by hand (RFC 1951 3.2.5-3.2.6: fixed codes are 8 bits for
# bytes 0..143, 7 bits for end-of-block and length codes 256..279, 5 bits for
# distances; one final block costs 3 header bits; a stored block is n+5).
HAND = [
    (b"", 2, "fixed"),          # 3 + 7 (end of block) = 10 bits
    (b"a", 3, "fixed"),         # 3 + 8 + 7 = 18 bits
    (b"abcabc", 8, "fixed"),    # no match: the only source is position 0 -> 6 literals: 3+48+7 = 58 bits
    (b"xabcabc", 7, "fixed"),   # 4 literals + (len 3: code 257, dist 3: code 2): 3+32+7+5+7 = 54 bits
    (b"abcdabcd", 8, "fixed"),  # 'a' at 4 would copy position 0 -> literal; 'bcd' copies position 1:
                                # 5 literals + len 3 + dist 4 (code 3): 3+40+7+5+7 = 62 bits
]


@pytest.mark.parametrize("x,nbytes,kind", HAND)
def test_hand_derived_sizes(x, nbytes, kind):
    raw, k = deflate1.deflate1_raw(x)
    assert len(raw) == nbytes
    assert k == kind
    assert raw == _zraw(x)


def test_incompressible_block_is_stored():
    # 64 bytes that never repeat a 3-byte string and use bytes >= 144
    # (9-bit fixed codes): fixed = 3+64*9+7 > stored = 64+5 bytes.
    x = bytes(range(144, 208))
    raw, k = deflate1.deflate1_raw(x)
    assert k == "stored" and len(raw) == 69


def test_gzip_framing_adds_18_bytes():
    rnd = random.Random(3)
    for _ in range(200):
        x = bytes(rnd.choice(b"abcde fgh") for _ in range(rnd.choice([16, 64, 128])))
        assert len(gzip.compress(x, compresslevel=1, mtime=0)) == deflate1.gzip1_len(x)
        assert deflate1.gzip1_len(x) == len(deflate1.deflate1_raw(x)[0]) + 18


def _families(rnd, b):
    words = [bytes(rnd.choice(b"abcdefghijklmnopqrstuvwxyz") for _ in range(rnd.randint(2, 5)))
             for _ in range(16)]
    yield "uniform", bytes(rnd.getrandbits(8) for _ in range(b))
    yield "printable", bytes(rnd.randint(32, 126) for _ in range(b))
    ph = b" ".join(rnd.choice(words) for _ in range(rnd.randint(1, 3))) + b" "
    yield "phrase", (ph * (b // len(ph) + 2))[:b]
    yield "run", bytes([rnd.randrange(256)]) * b
    yield "small_alphabet", bytes(rnd.randint(0, 3) for _ in range(b))
    x = bytearray(rnd.randint(97, 100) for _ in range(b))
    z = rnd.randint(0, b)
    x[z:] = bytes(b - z)
    yield "zero_tail", bytes(x)
    # repeats of the string at position 0 (which can never be a match source)
    head = bytes(rnd.randint(97, 99) for _ in range(rnd.randint(3, 6)))
    yield "repeat_pos0", (head * (b // len(head) + 1))[:b]
    # mixed 32-byte segments like the workloads, at this block size
    seg = bytearray()
    while len(seg) < b:
        seg += (bytes(rnd.randint(32, 126) for _ in range(32)) if rnd.random() < 0.4
                else (ph * 8)[:32])
    yield "segments", bytes(seg[:b])


@pytest.mark.parametrize("b", [16, 32, 64, 128, 256, 1024, 4096])
def test_byte_exact_with_zlib(b):
    rnd = random.Random(1000 + b)
    reps = {16: 3000, 32: 3000, 64: 2000, 128: 1500, 256: 400, 1024: 60, 4096: 12}[b]
    kinds = set()
    for _ in range(reps):
        for fam, x in _families(rnd, b):
            raw, k = deflate1.deflate1_raw(x)
            kinds.add(k)
            assert raw == _zraw(x), (fam, b, x.hex())
    if b >= 64:
        assert kinds == {"stored", "fixed", "dynamic"}


def test_round_trip_inflate():
    rnd = random.Random(11)
    for _ in range(2000):
        b = rnd.choice([16, 32, 64, 128, 300, 777])
        for _, x in _families(rnd, b):
            raw, _ = deflate1.deflate1_raw(x)
            assert zlib.decompress(raw, -15) == x


def _overflow_fixture():
    rows = []
    with open(os.path.join(HERE, "golden", "code_length_overflow.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            b, seed, hx = line.split()
            rows.append((int(b), bytes.fromhex(hx)))
    return rows


def test_code_length_tree_overflow_repair():
    rows = _overflow_fixture()
    assert len(rows) >= 8
    dynamic = 0
    for b, x in rows:
        assert len(x) == b
        # the unclamped code-length tree is deeper than 7 bits ...
        assert deflate1.tree_depths(x)[2] > 7
        # ... and the stream matches zlib: the repaired lengths decide the
        # block type, and a dynamic block sends them
        raw, k = deflate1.deflate1_raw(x)
        dynamic += k == "dynamic"
        assert raw == _zraw(x)
    assert dynamic >= 3


def test_batch_driver_matches_single_calls():
    rnd = np.random.default_rng(5)
    data = rnd.integers(97, 101, size=(3, 512), dtype=np.uint8)
    data[1, 100:300] = rnd.integers(32, 127, size=200)
    for b in (16, 64, 128):
        for nt in (1, 4):
            got = deflate1.block_lengths(data, b, nthreads=nt)
            want = [[len(gzip.compress(bytes(data[s, i * b:(i + 1) * b]), 1, mtime=0))
                     for i in range(512 // b)] for s in range(3)]
            assert got.tolist() == want


def test_size_limits():
    with pytest.raises(ValueError):
        deflate1.deflate1_raw(bytes(16384))
    raw, _ = deflate1.deflate1_raw(bytes(range(256)) * 63 + bytes(255))  # 16383 bytes
    assert raw == _zraw(bytes(range(256)) * 63 + bytes(255))
