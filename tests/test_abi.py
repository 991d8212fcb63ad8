"""The C ABI on the host (no GPU needed): the library loads, exports every
function include/gsa.h declares, and rejects bad arguments before launching
anything."""
import ctypes
import os
import re

import pytest

import content_adaptive_block_b200 as gsa
from content_adaptive_block_b200 import build as gsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    gsa_build.build()
    return gsa.library()


def _declared():
    import glob
    src = "".join(open(p).read() for p in sorted(glob.glob(os.path.join(ROOT, "include", "*.h"))))
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gsa_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_path(lib):
    names = _declared()
    for fn in ("gsa_block_lengths", "gsa_literal_flags", "gsa_build_block_csr", "gsa_mask_pipeline",
               "gsa_build_fixed_csr", "gsa_attn_fwd",
               "gsa_attn_bwd", "gsa_csr_capacity", "gsa_attn_bwd_workspace", "gsa_device_error",
               "gsa_status_string", "gsa_lm_block_workspace", "gsa_lm_block_fwd", "gsa_lm_block_bwd"):
        assert fn in names


def test_every_declared_symbol_is_exported(lib):
    for fn in _declared():
        assert hasattr(lib, fn), fn


def test_status_strings(lib):
    for code in range(6):
        assert gsa.gsa_status_string(code)
    assert gsa.gsa_status_string(99) == "unknown status"


def test_csr_capacity(lib):
    assert gsa.gsa_csr_capacity(1) == 1
    assert gsa.gsa_csr_capacity(128) == 128 * 129 // 2
    assert gsa.gsa_csr_capacity(0) == 0


NULL = ctypes.c_void_p(0)
FAKE = ctypes.c_void_p(0x1000)   # never dereferenced: every call below fails its host checks


def test_block_lengths_rejects_bad_arguments(lib):
    f = lib.gsa_block_lengths
    assert f(NULL, 1, 64, 64, FAKE, NULL) == 1
    assert f(FAKE, 1, 64, 64, NULL, NULL) == 1
    assert f(FAKE, 0, 64, 64, FAKE, NULL) == 1     # no samples
    assert f(FAKE, 1, 100, 64, FAKE, NULL) == 1    # L not a multiple of b
    assert f(FAKE, 1, 64, 0, FAKE, NULL) == 1      # b = 0
    assert f(FAKE, 1, 512, 256, FAKE, NULL) == 1   # b above the maximum
    assert f(FAKE, 1, 32, 64, FAKE, NULL) == 1     # L < b


def test_literal_flags_rejects_bad_arguments(lib):
    f = lib.gsa_literal_flags
    assert f(NULL, 1, 4, FAKE, NULL) == 1
    assert f(FAKE, 1, 4, NULL, NULL) == 1
    assert f(FAKE, 0, 4, FAKE, NULL) == 1
    assert f(FAKE, 1, 0, FAKE, NULL) == 1


def _csr(B=1, n=4, cap=None, classes=7):
    p = 0x1000
    return gsa._Csr(B, n, 0, classes, gsa.gsa_csr_capacity(n) if cap is None else cap, p, p, p, p, p, p)


def test_build_csr_rejects_bad_arguments(lib):
    f = lib.gsa_build_block_csr
    c = _csr()
    assert f(NULL, 1, NULL, 0, ctypes.byref(c), NULL) == 1
    assert f(FAKE, -1, NULL, 0, ctypes.byref(c), NULL) == 1          # negative window
    c0 = _csr(B=0)
    assert f(FAKE, 1, NULL, 0, ctypes.byref(c0), NULL) == 1
    small = _csr(n=8, cap=10)
    assert f(FAKE, 1, NULL, 0, ctypes.byref(small), NULL) == 3       # capacity
    nul = _csr()
    nul.q_order = None
    assert f(FAKE, 1, NULL, 0, ctypes.byref(nul), NULL) == 1
    hc = (ctypes.c_uint8 * 3)(0, 3, 1)
    assert f(FAKE, 1, ctypes.cast(hc, ctypes.c_void_p), 3, ctypes.byref(c), NULL) == 1   # class 3
    hc = (ctypes.c_uint8 * 1)(0)
    assert f(FAKE, 1, ctypes.cast(hc, ctypes.c_void_p), 0, ctypes.byref(c), NULL) == 1   # H = 0


def test_attention_rejects_heads_of_classes_not_built(lib):
    # lists of the local class only (classes = 0b001): a literal head is refused before any launch
    c = _csr(B=1, n=4, classes=1)
    hc = (ctypes.c_uint8 * 2)(0, 1)
    d = gsa._AttnDesc(1, 2, 256, 64, 64, 1, 0.0, ctypes.cast(hc, ctypes.c_void_p))
    p = FAKE
    assert lib.gsa_attn_fwd(p, p, p, ctypes.byref(c), ctypes.byref(d), p, p, NULL) == 1
    hc[1] = 0
    c.classes = 0
    assert lib.gsa_attn_fwd(p, p, p, ctypes.byref(c), ctypes.byref(d), p, p, NULL) == 1


def test_build_fixed_csr_rejects_bad_arguments(lib):
    f = lib.gsa_build_fixed_csr
    c = _csr(B=2, n=8)
    # kind, w, g, r, rnd, csr, stream
    assert f(2, 1, 1, 0, NULL, ctypes.byref(c), NULL) == 1            # unknown kind
    assert f(-1, 1, 1, 0, NULL, ctypes.byref(c), NULL) == 1
    assert f(0, -1, 1, 0, NULL, ctypes.byref(c), NULL) == 1           # negative window
    assert f(0, 1, -1, 0, NULL, ctypes.byref(c), NULL) == 1           # negative globals
    assert f(1, 1, 1, -1, FAKE, ctypes.byref(c), NULL) == 1           # negative random count
    assert f(1, 1, 1, 3, NULL, ctypes.byref(c), NULL) == 1            # BigBird picks without words
    assert f(0, 1, 1, 0, NULL, None, NULL) == 1                       # no csr
    assert f(1, 1, 1, 9, FAKE, ctypes.byref(c), NULL) == 2            # above GSA_MAX_RANDOM_BLOCKS
    big = _csr(B=1, n=8193)
    assert f(0, 1, 1, 0, NULL, ctypes.byref(big), NULL) == 2          # above GSA_MAX_FIXED_BLOCKS
    small = _csr(B=2, n=8, cap=10)
    assert f(0, 1, 1, 0, NULL, ctypes.byref(small), NULL) == 3        # capacity
    nul = _csr(B=2, n=8)
    nul.row_idx = None
    assert f(0, 1, 1, 0, NULL, ctypes.byref(nul), NULL) == 1


def _lm(B=2, L=1024, D=256, H=4, F=512, b=64, classes=(0, 0, 1, 2), eps=1e-5):
    hc = (ctypes.c_uint8 * len(classes))(*classes)
    return gsa._LmDesc(B, L, D, H, F, b, ctypes.cast(hc, ctypes.c_void_p), eps), hc


def test_lm_block_rejects_bad_arguments(lib):
    gsa._lm_fns()
    ws = lib.gsa_lm_block_workspace
    d, k0 = _lm()
    need = ws(ctypes.byref(d))
    assert need > 2 * 1024 * (22 * 256 + 6 * 512)
    for bad in (dict(D=192), dict(H=3, classes=(0, 0, 1)), dict(b=32), dict(L=1000), dict(F=500),
                dict(classes=(0, 0, 1, 3)), dict(eps=0.0), dict(B=0)):
        bd, kb = _lm(**bad)
        assert ws(ctypes.byref(bd)) == 0, bad
    c = _csr(B=2, n=16)
    w = gsa._LmPtrs(*([0x1000] * 9))
    g = gsa._LmPtrs(*([0x1000] * 9))
    f, fb = lib.gsa_lm_block_fwd, lib.gsa_lm_block_bwd
    assert f(FAKE, ctypes.byref(w), ctypes.byref(c), ctypes.byref(d), FAKE, FAKE, need - 1, NULL) == 3   # capacity
    assert f(NULL, ctypes.byref(w), ctypes.byref(c), ctypes.byref(d), FAKE, FAKE, need, NULL) == 1
    assert f(FAKE, ctypes.byref(w), ctypes.byref(c), ctypes.byref(d), NULL, FAKE, need, NULL) == 1
    wn = gsa._LmPtrs(*([0x1000] * 8 + [0]))
    assert f(FAKE, ctypes.byref(wn), ctypes.byref(c), ctypes.byref(d), FAKE, FAKE, need, NULL) == 1
    big, kg = _lm(D=2304, H=36, classes=(0,) * 36)
    assert f(FAKE, ctypes.byref(w), ctypes.byref(c), ctypes.byref(big), FAKE, FAKE, need, NULL) == 2   # D > 2048
    assert fb(FAKE, ctypes.byref(w), ctypes.byref(c), ctypes.byref(d), FAKE, ctypes.byref(g), FAKE, need - 1,
              NULL) == 3
    assert fb(FAKE, ctypes.byref(w), ctypes.byref(c), ctypes.byref(d), NULL, ctypes.byref(g), FAKE, need,
              NULL) == 1
    gn = gsa._LmPtrs(*([0] + [0x1000] * 8))
    assert fb(FAKE, ctypes.byref(w), ctypes.byref(c), ctypes.byref(d), FAKE, ctypes.byref(gn), FAKE, need,
              NULL) == 1


def test_mask_pipeline_rejects_bad_arguments(lib):
    f = lib.gsa_mask_pipeline
    c = _csr(B=2, n=8)
    # bytes, B, L, b, w, head_classes, H, lengths, flags, csr, counter, stream; 2 samples x 512 bytes, b=64
    def call(**kw):
        a = dict(bytes=FAKE, B=2, L=512, b=64, w=1, hc=NULL, H=0, lengths=FAKE, flags=FAKE, csr=ctypes.byref(c),
                 counter=FAKE)
        a.update(kw)
        return f(a["bytes"], a["B"], a["L"], a["b"], a["w"], a["hc"], a["H"], a["lengths"], a["flags"], a["csr"],
                 a["counter"], NULL)
    for name in ("bytes", "lengths", "flags", "counter"):       # null device pointers
        assert call(**{name: NULL}) == 1, name
    assert call(w=-1) == 1                                       # negative window
    assert call(L=500) == 1                                      # L % b
    assert call(B=3) == 1                                        # csr->B != B
    assert call(L=1024) == 1                                     # csr->nblk != L / b
    hc = (ctypes.c_uint8 * 2)(0, 5)
    assert call(hc=ctypes.cast(hc, ctypes.c_void_p), H=2) == 1   # a class outside 0..2
    big = _csr(B=1, n=2048)
    assert call(B=1, L=2048 * 16, b=16, csr=ctypes.byref(big)) == 2   # beyond one launch
    small = _csr(B=2, n=8, cap=10)
    assert call(csr=ctypes.byref(small)) == 3                    # capacity


def _desc(B=1, H=4, L=256, d=64, b=64, dtype=1, classes=(0, 0, 1, 2), scale=0.0):
    hc = (ctypes.c_uint8 * len(classes))(*classes)
    return gsa._AttnDesc(B, H, L, d, b, dtype, scale, ctypes.cast(hc, ctypes.c_void_p)), hc


def test_attn_fwd_rejects_bad_arguments(lib):
    f = lib.gsa_attn_fwd
    c = _csr(n=4)
    d, keep = _desc()
    assert f(NULL, FAKE, FAKE, ctypes.byref(c), ctypes.byref(d), FAKE, FAKE, NULL) == 1
    bad_l, k1 = _desc(L=200)                                 # L != nblk * b
    assert f(FAKE, FAKE, FAKE, ctypes.byref(c), ctypes.byref(bad_l), FAKE, FAKE, NULL) == 1
    bad_c, k2 = _desc(classes=(0, 0, 1, 3))                  # class outside 0..2
    assert f(FAKE, FAKE, FAKE, ctypes.byref(c), ctypes.byref(bad_c), FAKE, FAKE, NULL) == 1
    bad_b, k3 = _desc(B=2)                                   # batch disagrees with the lists
    assert f(FAKE, FAKE, FAKE, ctypes.byref(c), ctypes.byref(bad_b), FAKE, FAKE, NULL) == 1
    c32 = _csr(n=8)
    d32, k4 = _desc(L=256, b=32)                             # bf16 path needs b = 64
    assert f(FAKE, FAKE, FAKE, ctypes.byref(c32), ctypes.byref(d32), FAKE, FAKE, NULL) == 2
    dd, k5 = _desc(d=96)                                     # head dim not implemented
    assert f(FAKE, FAKE, FAKE, ctypes.byref(c), ctypes.byref(dd), FAKE, FAKE, NULL) == 2
    small = _csr(n=4, cap=3)
    assert f(FAKE, FAKE, FAKE, ctypes.byref(small), ctypes.byref(d), FAKE, FAKE, NULL) == 3
    neg, k6 = _desc(scale=-1.0)
    assert f(FAKE, FAKE, FAKE, ctypes.byref(c), ctypes.byref(neg), FAKE, FAKE, NULL) == 1


def test_attn_layout_rejects_bad_strides(lib):
    f = lib.gsa_attn_fwd
    c = _csr(n=4)
    good = (3 * 256 * 4 * 64, 64, 3 * 4 * 64, 256 * 4 * 64, 64, 4 * 64)
    for i, bad in ((0, 12), (1, 0), (2, -64), (2, 32), (5, 8)):   # not a multiple of 8, <= 0, token stride < d
        s = list(good)
        s[i] = bad
        lay = gsa._AttnLayout(*s)
        d, keep = _desc()
        d.layout = ctypes.cast(ctypes.pointer(lay), ctypes.c_void_p)
        assert f(FAKE, FAKE, FAKE, ctypes.byref(c), ctypes.byref(d), FAKE, FAKE, NULL) == 1, (i, bad)
    lay = gsa._AttnLayout(*good)
    d32, keep = _desc(dtype=0)
    d32.layout = ctypes.cast(ctypes.pointer(lay), ctypes.c_void_p)
    assert f(FAKE, FAKE, FAKE, ctypes.byref(c), ctypes.byref(d32), FAKE, FAKE, NULL) == 2   # float32: dense only
    d, keep = _desc()
    odd = ctypes.c_void_p(0x1008)                                 # bf16 tensors must be 16-byte aligned
    assert f(odd, FAKE, FAKE, ctypes.byref(c), ctypes.byref(d), FAKE, FAKE, NULL) == 1


def test_attn_bwd_rejects_bad_arguments(lib):
    f = lib.gsa_attn_bwd
    c = _csr(n=4)
    d, keep = _desc()
    ws = lib.gsa_attn_bwd_workspace(ctypes.byref(d))
    rows = 1 * 4 * 256
    assert ws == 2 * 4 * ((rows + 63) // 64 * 64) + 256   # -D and -LSE log2(e) (float32 per row), then counters
    args = [FAKE] * 6
    assert f(*args[:5], NULL, ctypes.byref(c), ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, ws, NULL) == 1
    assert f(*args, ctypes.byref(c), ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, ws - 4, NULL) == 3
    d32, k2 = _desc(dtype=0, d=32)
    assert f(*args, ctypes.byref(c), ctypes.byref(d32), FAKE, FAKE, FAKE, FAKE, 1 << 20, NULL) == 2


def test_device_error_rejects_null(lib):
    assert lib.gsa_device_error(None, 0) == 1


def test_python_binding_refuses_cpu_tensors(lib):
    import torch
    with pytest.raises(ValueError):
        gsa.gsa_block_lengths(torch.zeros((1, 64), dtype=torch.uint8), 64)
    with pytest.raises(ValueError):
        gsa.gsa_literal_flags(torch.zeros((1, 4), dtype=torch.int32))


def test_binding_mirrors_every_header_function():
    """The Python binding exposes each C entry point of include/*.h under the
    same name (and lists it in __all__)."""
    import re
    import content_adaptive_block_b200 as gsa
    names = set()
    for h in ("gsa.h", "gsa_lm.h"):
        text = open(os.path.join(ROOT, "include", h)).read()
        names |= set(re.findall(r"^[A-Za-z_][\w \*]*?\b(gsa_\w+)\s*\(", text, re.M))
    assert len(names) >= 16, names
    for n in sorted(names):
        assert callable(getattr(gsa, n, None)), n
        assert n in gsa.__all__, n


def test_noalloc_max_rows_through_the_binding():
    import content_adaptive_block_b200 as gsa
    assert gsa.gsa_attn_bwd_noalloc_max_rows() == 1 << 21
