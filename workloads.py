"""Seeded synthetic inputs and the workload table.

This module only makes inputs: byte streams shaped like the byte-level text
the method is evaluated on, and N(0, 1) query/key/value/gradient tensors.  It
holds none of the method's arithmetic; both the CUDA path's tests and the
oracle draw their inputs from here.

Byte streams (stand-ins for raw UTF-8 book/wiki text, which is not available):
a sample is a run of 32-byte segments.  With probability f a segment is
high-entropy — 32 bytes drawn uniformly from printable ASCII 32..126 —
otherwise it repeats a phrase of 1–3 words (from a 16-word vocabulary of
2–5 lowercase letters drawn per sample), words joined and followed by a
space, to fill the 32 bytes.  The long-context workload instead repeats one
16-byte phrase per sample, so that every untouched 64-byte block compresses
the same and only about sqrt(N) blocks rise above the mean.
"""
from __future__ import annotations

import dataclasses

import numpy as np

SEGMENT = 32
LOCAL, LITERAL, HYBRID = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    S: int                 # batch (samples)
    L: int                 # bytes (= tokens) per sample
    b: int                 # block size in bytes
    w: int                 # local window in blocks
    H: int                 # heads
    d: int                 # head dimension
    dtype: str             # "f32" or "bf16"
    backward: bool
    entropy: tuple         # ("fixed", f) | ("uniform", lo, hi) | ("period16", f)
    salt: int

    @property
    def N(self) -> int:
        return self.L // self.b

    def head_classes(self) -> np.ndarray:
        """Half local, a quarter literal, a quarter hybrid, in that order."""
        h = np.empty(self.H, dtype=np.uint8)
        h[: self.H // 2] = LOCAL
        h[self.H // 2: 3 * self.H // 4] = LITERAL
        h[3 * self.H // 4:] = HYBRID
        return h


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", S=1, L=256, b=16, w=1, H=4, d=32, dtype="f32",
                          backward=False, entropy=("fixed", 0.5), salt=1),
    "b8_4k": Workload("b8_4k", S=8, L=4096, b=64, w=2, H=12, d=64, dtype="bf16",
                      backward=False, entropy=("uniform", 0.2, 0.6), salt=2),
    "b8_8k": Workload("b8_8k", S=8, L=8192, b=64, w=2, H=12, d=64, dtype="bf16",
                      backward=True, entropy=("uniform", 0.2, 0.6), salt=3),
    "b1_64k": Workload("b1_64k", S=1, L=65536, b=64, w=4, H=16, d=128, dtype="bf16",
                       backward=True, entropy=("period16", 0.015), salt=4),
}


def mask_sweep(b: int, f: float) -> Workload:
    """Mask-stage sweep point: 256 samples of 8192 bytes, window 2."""
    return Workload(f"mask_b{b}_f{f}", S=256, L=8192, b=b, w=2, H=12, d=64, dtype="bf16",
                    backward=False, entropy=("fixed", f), salt=5 + b * 1000 + int(round(f * 100)))


MASK_SWEEP = [(b, f) for b in (32, 64, 128) for f in (0.05, 0.3, 0.7)]


def seq_sweep(L: int) -> Workload:
    """Sequence-length sweep point: the 8x8K configuration (b=64, w=2, 12
    heads 6/3/3, d=64, bf16, forward and backward, entropy U[0.2, 0.6]) at
    length L with the batch shrunk so that S * L = 65536 bytes per step."""
    return Workload(f"seq_{L // 1024}k", S=max(1, 65536 // L), L=L, b=64, w=2, H=12, d=64, dtype="bf16",
                    backward=True, entropy=("uniform", 0.2, 0.6), salt=7 + L)


SEQ_SWEEP = [4096, 8192, 16384, 32768, 65536]


# Fixed comparison masks at block 64 (the 8x8K shape: 128 blocks per sample),
# with the published defaults of each pattern read at block granularity:
# BigBird — a 3-block sliding window (w = 1), 2 global blocks, 3 random
# blocks per query block; Longformer — a 512-token window (256 tokens, w = 4
# blocks, each side) and one global block.
FIXED_MASKS = {
    "bigbird": dict(kind=1, w=1, g=2, r=3),
    "longformer": dict(kind=0, w=4, g=1, r=0),
}


def random_words(S: int, n: int, r: int, seed: int = 0) -> np.ndarray:
    """uint32 [S, n, r] uniform words: the random draws of BigBird's picks."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 0xB16B, S, n, r])))
    return rng.integers(0, 2**32, size=(S, n, r), dtype=np.uint64).astype(np.uint32)


# One ByteLM block at the width of a 12-block, ~85M-weight byte LM (the
# paper's 92M / 8K model class): D = 768, 12 heads of 64, MLP 3072, on the
# 8x8K bench batch; the small shape spans several 128-row tiles with a ragged
# tail (17 blocks per sample) for exact parity.
LM_BLOCK = dict(D=768, H=12, F=3072)
LM_BLOCK_SMALL = dict(S=2, L=17 * 64, D=256, H=4, F=512, w=2)


def lm_weights(D: int, F: int, seed: int = 0, device="cpu", std: float = 0.02):
    """Random-init weights of one block: matrices ~ N(0, std^2) in bf16, the
    embedding ~ N(0, 1) in bf16, LayerNorm gains ~ 1 + N(0, 0.1^2) and biases
    ~ N(0, 0.1^2) in float32 (perturbed so their gradients are exercised)."""
    import torch
    g = torch.Generator(device="cpu")
    g.manual_seed(9_000_011 + seed)

    def n(*shape, s=1.0):
        return torch.randn(*shape, generator=g, dtype=torch.float32) * s

    w = {"emb": n(256, D).bfloat16(), "ln1_g": 1 + n(D, s=0.1), "ln1_b": n(D, s=0.1),
         "w_qkv": n(3 * D, D, s=std).bfloat16(), "w_o": n(D, D, s=std).bfloat16(),
         "ln2_g": 1 + n(D, s=0.1), "ln2_b": n(D, s=0.1),
         "w_1": n(F, D, s=std).bfloat16(), "w_2": n(D, F, s=std).bfloat16()}
    return {k: v.to(device) for k, v in w.items()}


def _rng(seed: int, salt: int, s: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, salt, s])))


def _vocab(rng, n=16):
    words = []
    for _ in range(n):
        ln = int(rng.integers(2, 6))
        words.append(bytes(rng.integers(ord("a"), ord("z") + 1, size=ln).astype(np.uint8)))
    return words


def _phrase_segment(rng, vocab) -> bytes:
    k = int(rng.integers(1, 4))
    idx = rng.integers(0, len(vocab), size=k)
    phrase = b" ".join(vocab[i] for i in idx) + b" "
    return (phrase * (SEGMENT // len(phrase) + 1))[:SEGMENT]


def _noise_segment(rng) -> bytes:
    return bytes(rng.integers(32, 127, size=SEGMENT).astype(np.uint8))


def sample_bytes(L: int, entropy: tuple, seed: int, salt: int, s: int) -> np.ndarray:
    """One sample of L bytes (L a multiple of 32)."""
    if L % SEGMENT:
        raise ValueError("L must be a multiple of 32")
    rng = _rng(seed, salt, s)
    vocab = _vocab(rng)
    kind = entropy[0]
    if kind == "fixed":
        f = float(entropy[1])
    elif kind == "uniform":
        f = float(rng.uniform(entropy[1], entropy[2]))
    elif kind == "period16":
        f = float(entropy[1])
    else:
        raise ValueError(kind)
    if kind == "period16":
        words = b" ".join(vocab) + b" "
        period = (words * 2)[:16]
        fill = period * (SEGMENT // 16)
    out = bytearray()
    for _ in range(L // SEGMENT):
        if rng.random() < f:
            out += _noise_segment(rng)
        elif kind == "period16":
            out += fill
        else:
            out += _phrase_segment(rng, vocab)
    return np.frombuffer(bytes(out), dtype=np.uint8)


def batch_bytes(wl: Workload, seed: int = 0) -> np.ndarray:
    """uint8 [S, L] byte streams of a workload."""
    return np.stack([sample_bytes(wl.L, wl.entropy, seed, wl.salt, s) for s in range(wl.S)])


def custom_bytes(S: int, L: int, entropy: tuple, seed: int = 0, salt: int = 99) -> np.ndarray:
    return np.stack([sample_bytes(L, entropy, seed, salt, s) for s in range(S)])


def qkv(wl: Workload, seed: int = 0, device="cpu", grad: bool = False):
    """Q, K, V (and dO when grad) ~ N(0, 1), [S, H, L, d], in the workload's
    dtype, from a seeded torch generator on the given device."""
    import torch
    dt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    g = torch.Generator(device=device)
    g.manual_seed(1_000_003 * seed + wl.salt)
    shape = (wl.S, wl.H, wl.L, wl.d)
    out = [torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(dt) for _ in range(4 if grad else 3)]
    return tuple(out)


def random_tensors(shape, n, dtype, seed, device="cpu"):
    """n tensors ~ N(0, 1) of a shape, seeded."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return tuple(torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(dtype) for _ in range(n))
