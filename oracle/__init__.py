"""ORACLE — test infrastructure only.

A plain, slow, obviously correct CPU statement of what gzip-guided sparse
attention computes, written from the pages that describe it (Gzip-guided
Sparse Attention, daiwk.github.io reproduction of arXiv 2607.21752, section
"核心公式" and "背景与主要改动"; the abstract page "Parameter-free Adaptive Sparse
Attention via Compression-Based Content Selection").

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never links, loads or
calls it, and it shares no code with the CUDA library.

Modules
-------
deflate1   per-block gzip level-1 compressed length (a from-scratch DEFLATE
           compressor in plain C, loaded through ctypes)
flags      literal flags  l_i = 1[r_i > mean r]  in exact rational arithmetic
mask       the block mask M = M_lit ∪ M_local ∪ I intersected with causality,
           per head class, and its row / column lists
attention  masked softmax attention and its gradient in float64
"""

from . import deflate1, flags, mask, attention  # noqa: F401

LOCAL, LITERAL, HYBRID = 0, 1, 2
