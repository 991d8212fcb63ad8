"""ORACLE — test infrastructure only.  ctypes front end of deflate1.c.

Gzip-guided Sparse Attention (daiwk.github.io), section "核心公式", r_i
equation: the compression ratio of block i is |gzip(x_{ib:(i+1)b})| / b, each
block compressed on its own at gzip level 1 (flowchart node "gzip level-1 per
block").  This module returns |gzip(block)| in bytes; the division by b is
left to the flag rule (it is a common factor of every block of a sample).

The shared object is built from deflate1.c with the host C compiler the first
time it is needed (or by ``build()``), into ``oracle/_build/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "deflate1.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle_deflate1.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile deflate1.c into oracle/_build/liboracle_deflate1.so."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-o", tmp,
                        _SRC, "-lpthread"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_deflate1_raw.restype = ctypes.c_long
            lib.oracle_deflate1_raw.argtypes = [ctypes.c_void_p, ctypes.c_long, ctypes.c_void_p,
                                                ctypes.c_long, ctypes.POINTER(ctypes.c_int)]
            lib.oracle_deflate1_tree_depths.restype = ctypes.c_long
            lib.oracle_deflate1_tree_depths.argtypes = [ctypes.c_void_p, ctypes.c_long,
                                                        ctypes.POINTER(ctypes.c_int)]
            lib.oracle_gzip1_len.restype = ctypes.c_long
            lib.oracle_gzip1_len.argtypes = [ctypes.c_void_p, ctypes.c_long]
            lib.oracle_gzip1_block_lengths.restype = ctypes.c_int
            lib.oracle_gzip1_block_lengths.argtypes = [ctypes.c_void_p, ctypes.c_long, ctypes.c_long,
                                                       ctypes.c_long, ctypes.c_void_p, ctypes.c_int]
            _lib = lib
    return _lib


BLOCK_KINDS = ("stored", "fixed", "dynamic")


def deflate1_raw(x: bytes) -> tuple[bytes, str]:
    """The raw DEFLATE stream of x at level 1 and its block kind."""
    lib = _load()
    x = bytes(x)
    cap = len(x) + 64
    out = ctypes.create_string_buffer(cap)
    kind = ctypes.c_int(-1)
    n = lib.oracle_deflate1_raw(x, len(x), out, cap, ctypes.byref(kind))
    if n < 0:
        raise ValueError(f"oracle_deflate1_raw failed ({n}) for {len(x)} bytes")
    return out.raw[:n], BLOCK_KINDS[kind.value]


def gzip1_len(x: bytes) -> int:
    """|gzip(x)| at level 1: 10-byte header + raw DEFLATE + 8-byte trailer."""
    lib = _load()
    x = bytes(x)
    n = lib.oracle_gzip1_len(x, len(x))
    if n < 0:
        raise ValueError(f"oracle_gzip1_len failed ({n})")
    return int(n)


def tree_depths(x: bytes) -> tuple[int, int, int]:
    """Deepest leaf of the literal/length, distance and code-length trees
    before the 15/15/7-bit limits are applied."""
    lib = _load()
    x = bytes(x)
    d = (ctypes.c_int * 3)()
    if lib.oracle_deflate1_tree_depths(x, len(x), d) < 0:
        raise ValueError("oracle_deflate1_tree_depths failed")
    return int(d[0]), int(d[1]), int(d[2])


def block_lengths(data: np.ndarray, b: int, nthreads: int = 1) -> np.ndarray:
    """lengths[s, i] = |gzip level 1 of data[s, i*b:(i+1)*b]|, int32 [S, L/b].

    data is a uint8 array [S, L] (or [L]).  Blocks are independent; nthreads
    POSIX threads split the loop over them.
    """
    lib = _load()
    a = np.ascontiguousarray(data, dtype=np.uint8)
    if a.ndim == 1:
        a = a[None, :]
    S, L = a.shape
    if b <= 0 or L % b != 0:
        raise ValueError("L must be a multiple of b")
    out = np.empty((S, L // b), dtype=np.int32)
    rc = lib.oracle_gzip1_block_lengths(a.ctypes.data, S, L, b, out.ctypes.data, int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_gzip1_block_lengths failed ({rc})")
    return out
