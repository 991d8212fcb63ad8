"""Gzip-guided sparse attention hot path on B200 — Python binding of libgsa.

Thin ctypes marshalling over the C ABI in include/gsa.h: every function here
checks tensor placement/dtype/shape, builds the C argument structs and calls
the library function of the same name.  All arithmetic runs in the CUDA
kernels of libgsa.so; there is no CPU fallback.  PyTorch only provides the
device memory and the stream.

Pipeline (Gzip-guided Sparse Attention, daiwk.github.io, "核心公式"):
    lengths = gsa_block_lengths(bytes, b)            # |gzip(block)| per block
    flags   = gsa_literal_flags(lengths)             # l_i = 1[r_i > mean r]
    csr     = gsa_build_block_csr(flags, w)          # mask lists per head class
    o, lse  = gsa_attn_fwd(q, k, v, csr, head_classes, b)
    dq, dk, dv = gsa_attn_bwd(q, k, v, o, lse, do, csr, head_classes, b)
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "GsaError", "BlockCsr", "HEAD_LOCAL", "HEAD_LITERAL", "HEAD_HYBRID",
    "gsa_block_lengths", "gsa_literal_flags", "gsa_build_block_csr", "gsa_build_fixed_csr", "gsa_mask_pipeline",
    "gsa_csr_capacity", "gsa_attn_fwd", "gsa_attn_bwd", "gsa_attn_bwd_workspace", "gsa_attn_bwd_noalloc",
    "gsa_attn_bwd_noalloc_max_rows", "gsa_lm_block_workspace", "gsa_lm_block_fwd", "gsa_lm_block_bwd",
    "gsa_lm_gemm", "gsa_lm_gemm_workspace",
    "gsa_device_error", "gsa_status_string", "library", "library_path",
]

HEAD_LOCAL, HEAD_LITERAL, HEAD_HYBRID = 0, 1, 2
GSA_F32, GSA_BF16 = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))
# GSA_LIBRARY_PATH may point at another build of the same library (tuning).
_LIB_PATH = os.environ.get("GSA_LIBRARY_PATH") or os.path.join(_HERE, "lib", "libgsa.so")
_lib = None


class GsaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {gsa_status_string(status)} (status {status})")
        self.status = status


class _Csr(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("nblk", ctypes.c_int32), ("w", ctypes.c_int32),
        ("classes", ctypes.c_int32), ("capacity", ctypes.c_int64),
        ("row_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p),
        ("col_ptr", ctypes.c_void_p), ("row_idx", ctypes.c_void_p),
        ("q_order", ctypes.c_void_p), ("k_order", ctypes.c_void_p),
    ]


class _AttnLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("qkv_s", "qkv_h", "qkv_l", "o_s", "o_h", "o_l")]


class _AttnDesc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("L", ctypes.c_int64),
        ("d", ctypes.c_int32), ("b", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("scale", ctypes.c_float), ("head_classes", ctypes.c_void_p),
        ("layout", ctypes.c_void_p),
    ]


def library_path() -> str:
    return _LIB_PATH


def library():
    """Load libgsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libgsa.so is not built ({_LIB_PATH}); run "
                               "`python -m content_adaptive_block_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        lib.gsa_block_lengths.argtypes = [vp, i32, i64, i32, vp, vp]
        lib.gsa_literal_flags.argtypes = [vp, i32, i32, vp, vp]
        lib.gsa_build_block_csr.argtypes = [vp, i32, vp, i32, ctypes.POINTER(_Csr), vp]
        lib.gsa_mask_pipeline.argtypes = [vp, i32, i64, i32, i32, vp, i32, vp, vp, ctypes.POINTER(_Csr), vp, vp]
        lib.gsa_build_fixed_csr.argtypes = [i32, i32, i32, i32, vp, ctypes.POINTER(_Csr), vp]
        lib.gsa_csr_capacity.argtypes = [i32]
        lib.gsa_csr_capacity.restype = i64
        lib.gsa_attn_fwd.argtypes = [vp, vp, vp, ctypes.POINTER(_Csr), ctypes.POINTER(_AttnDesc), vp, vp, vp]
        lib.gsa_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.POINTER(_Csr), ctypes.POINTER(_AttnDesc),
                                     vp, vp, vp, vp, ctypes.c_size_t, vp]
        lib.gsa_attn_bwd_workspace.argtypes = [ctypes.POINTER(_AttnDesc)]
        lib.gsa_attn_bwd_workspace.restype = ctypes.c_size_t
        lib.gsa_device_error.argtypes = [ctypes.POINTER(i32), i32]
        lib.gsa_status_string.argtypes = [ctypes.c_int]
        lib.gsa_status_string.restype = ctypes.c_char_p
        for fn in ("gsa_block_lengths", "gsa_literal_flags", "gsa_build_block_csr", "gsa_mask_pipeline",
                   "gsa_build_fixed_csr", "gsa_attn_fwd", "gsa_attn_bwd", "gsa_device_error"):
            getattr(lib, fn).restype = ctypes.c_int
        _lib = lib
    return _lib


def gsa_status_string(status: int) -> str:
    return library().gsa_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != 0:
        raise GsaError(fn, status)


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _need(t: torch.Tensor, name: str, dtype=None, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


# ------------------------------------------------------------------ mask stage

def gsa_block_lengths(data: torch.Tensor, b: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """|gzip level 1| of every b-byte block of data (uint8 [B, L]) -> int32 [B, L/b]."""
    _need(data, "data", torch.uint8, 2)
    B, L = data.shape
    if out is None:
        out = torch.empty((B, L // b if b > 0 else 0), dtype=torch.int32, device=data.device)
    _need(out, "out", torch.int32)
    _check("gsa_block_lengths",
           library().gsa_block_lengths(_ptr(data), B, L, int(b), _ptr(out), _stream(stream)))
    return out


def gsa_literal_flags(lengths: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Literal flags (uint8 [B, nblk]) from per-block lengths (int32 [B, nblk])."""
    _need(lengths, "lengths", torch.int32, 2)
    B, n = lengths.shape
    if out is None:
        out = torch.empty((B, n), dtype=torch.uint8, device=lengths.device)
    _need(out, "out", torch.uint8)
    _check("gsa_literal_flags", library().gsa_literal_flags(_ptr(lengths), B, n, _ptr(out), _stream(stream)))
    return out


def gsa_csr_capacity(nblk: int) -> int:
    return int(library().gsa_csr_capacity(int(nblk)))


class BlockCsr:
    """Device buffers of the per-(sample, class) block lists (gsa_block_csr)."""

    def __init__(self, B: int, nblk: int, device, capacity: int | None = None):
        cap = gsa_csr_capacity(nblk) if capacity is None else int(capacity)
        i32 = dict(dtype=torch.int32, device=device)
        self.B, self.nblk, self.capacity, self.w = B, nblk, cap, -1
        self.classes = 0   # bitmask of the head classes whose lists were built
        self.row_ptr = torch.empty((B, 3, nblk + 1), **i32)
        self.col_idx = torch.empty((B, 3, cap), **i32)
        self.col_ptr = torch.empty((B, 3, nblk + 1), **i32)
        self.row_idx = torch.empty((B, 3, cap), **i32)
        self.q_order = torch.empty((B, 3, nblk), **i32)
        self.k_order = torch.empty((B, 3, nblk), **i32)

    def struct(self) -> _Csr:
        return _Csr(self.B, self.nblk, self.w, self.classes, self.capacity,
                    self.row_ptr.data_ptr(), self.col_idx.data_ptr(), self.col_ptr.data_ptr(),
                    self.row_idx.data_ptr(), self.q_order.data_ptr(), self.k_order.data_ptr())

    def stored(self, c: int) -> bool:
        """Whether class c's lists are in the buffers: a local class marked
        implicit (classes bit 3, written by gsa_mask_pipeline) is not stored;
        the attention kernels derive its lists from (nblk, w)."""
        return not (c == 0 and self.classes & 8)

    def rows(self, s: int, c: int) -> list:
        """Key-block list of every query block of (sample s, class c), on the host."""
        if not self.stored(c):
            raise ValueError("the local class's lists are implicit (not stored)")
        rp = self.row_ptr[s, c].cpu().tolist()
        ci = self.col_idx[s, c, : rp[-1]].cpu().tolist()
        return [ci[rp[i]: rp[i + 1]] for i in range(self.nblk)]

    def cols(self, s: int, c: int) -> list:
        if not self.stored(c):
            raise ValueError("the local class's lists are implicit (not stored)")
        cp = self.col_ptr[s, c].cpu().tolist()
        ri = self.row_idx[s, c, : cp[-1]].cpu().tolist()
        return [ri[cp[j]: cp[j + 1]] for j in range(self.nblk)]


def gsa_build_block_csr(flags: torch.Tensor, w: int, csr: BlockCsr | None = None, stream=None,
                        head_classes=None) -> BlockCsr:
    """Block lists of the mask from literal flags: for the classes in
    head_classes (one per head), or for all three classes when it is None."""
    _need(flags, "flags", torch.uint8, 2)
    B, n = flags.shape
    if csr is None:
        csr = BlockCsr(B, n, flags.device)
    st = csr.struct()
    hc, H = None, 0
    if head_classes is not None:
        H = len(head_classes)
        hc = (ctypes.c_uint8 * H)(*[int(c) for c in head_classes])
    _check("gsa_build_block_csr", library().gsa_build_block_csr(_ptr(flags), int(w),
                                                                 ctypes.cast(hc, ctypes.c_void_p) if hc else None,
                                                                 H, ctypes.byref(st), _stream(stream)))
    csr.w, csr.classes = st.w, st.classes
    return csr


GSA_FIXED_LONGFORMER, GSA_FIXED_BIGBIRD = 0, 1


def gsa_build_fixed_csr(kind: int, B: int, nblk: int, w: int, g: int, rnd: torch.Tensor | None = None,
                        device=None, csr: BlockCsr | None = None, stream=None) -> BlockCsr:
    """Block lists of a fixed comparison mask (GSA_FIXED_LONGFORMER: window w
    and g global blocks; GSA_FIXED_BIGBIRD: plus random key blocks from the
    uint32 words rnd [B, nblk, r]), the same in all three class slots."""
    r = 0
    if rnd is not None:
        _need(rnd, "rnd", torch.int32 if rnd.dtype == torch.int32 else torch.uint32, 3)
        if tuple(rnd.shape[:2]) != (B, nblk):
            raise ValueError("rnd must be [B, nblk, r]")
        r = int(rnd.shape[2])
        device = rnd.device if device is None else device
    if csr is None:
        csr = BlockCsr(B, nblk, device)
    st = csr.struct()
    _check("gsa_build_fixed_csr", library().gsa_build_fixed_csr(int(kind), int(w), int(g), r,
                                                                 _ptr(rnd) if rnd is not None else None,
                                                                 ctypes.byref(st), _stream(stream)))
    csr.w, csr.classes = st.w, st.classes
    return csr


def gsa_mask_pipeline(data: torch.Tensor, b: int, w: int, csr: BlockCsr | None = None,
                      lengths: torch.Tensor | None = None, flags: torch.Tensor | None = None,
                      counters: torch.Tensor | None = None, stream=None, head_classes=None):
    """lengths -> flags -> block lists in one launch; returns (lengths, flags, csr).
    The local class's lists are implicit: not stored (csr.classes bit 3), the
    attention kernels derive them from (nblk, w).  counters (int32,
    at least one element, zero, left zero by each call) may be passed to avoid
    allocating one per call."""
    _need(data, "data", torch.uint8, 2)
    B, L = data.shape
    n = L // b if b > 0 else 0
    if lengths is None:
        lengths = torch.empty((B, n), dtype=torch.int32, device=data.device)
    if flags is None:
        flags = torch.empty((B, n), dtype=torch.uint8, device=data.device)
    if csr is None:
        csr = BlockCsr(B, n, data.device)
    if counters is None:
        counters = torch.zeros(1, dtype=torch.int32, device=data.device)
    _need(lengths, "lengths", torch.int32)
    _need(flags, "flags", torch.uint8)
    _need(counters, "counters", torch.int32)
    st = csr.struct()
    hc, H = None, 0
    if head_classes is not None:
        H = len(head_classes)
        hc = (ctypes.c_uint8 * H)(*[int(c) for c in head_classes])
    _check("gsa_mask_pipeline", library().gsa_mask_pipeline(_ptr(data), B, L, int(b), int(w),
                                                             ctypes.cast(hc, ctypes.c_void_p) if hc else None, H,
                                                             _ptr(lengths), _ptr(flags), ctypes.byref(st),
                                                             _ptr(counters), _stream(stream)))
    csr.w, csr.classes = st.w, st.classes
    return lengths, flags, csr


# ------------------------------------------------------------------ attention

def _desc(q: torch.Tensor, b: int, head_classes, scale: float, o: torch.Tensor | None = None):
    """The call's descriptor; q (and o) may be strided [B, H, L, d] views with
    contiguous rows, which become the call's layout (None when dense)."""
    B, H, L, d = q.shape
    hc = (ctypes.c_uint8 * H)(*[int(c) for c in head_classes])
    dtype = GSA_F32 if q.dtype == torch.float32 else GSA_BF16
    keep = [hc]
    lay = None
    if not q.is_contiguous() or (o is not None and not o.is_contiguous()):
        so = o.stride() if o is not None else q.stride()
        lay = _AttnLayout(q.stride(0), q.stride(1), q.stride(2), so[0], so[1], so[2])
        keep.append(lay)
    desc = _AttnDesc(B, H, L, d, int(b), dtype, float(scale), ctypes.cast(hc, ctypes.c_void_p),
                     ctypes.cast(ctypes.pointer(lay), ctypes.c_void_p) if lay is not None else None)
    return desc, keep


def _need_rows(t: torch.Tensor, name: str, like: torch.Tensor):
    """A [B, H, L, d] CUDA tensor of like's dtype, shape and strides, d contiguous."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != like.dtype or t.dim() != 4 or tuple(t.shape) != tuple(like.shape):
        raise ValueError(f"{name} must be {like.dtype} of shape {tuple(like.shape)}")
    if t.stride(3) != 1 or t.stride() != like.stride():
        raise ValueError(f"{name} must have the strides of {like.stride()} with contiguous rows")


def gsa_attn_fwd(q, k, v, csr: BlockCsr, head_classes, b: int, scale: float = 0.0,
                 o: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """Block-sparse causal attention forward; q, k, v [B, H, L, d] (bf16 or
    float32), bf16 ones possibly strided views with contiguous rows (k and v
    with q's strides; o may have its own).  Returns (o, lse) with lse float32
    [B, H, L]."""
    if q.dtype == torch.float32:
        for name, t in (("q", q), ("k", k), ("v", v)):
            _need(t, name, q.dtype, 4)
    else:
        _need_rows(q, "q", q)
        _need_rows(k, "k", q)
        _need_rows(v, "v", q)
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k and v must have the same shape")
    if len(head_classes) != q.shape[1]:
        raise ValueError("one head class per head")
    if o is None:
        o = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    if q.dtype == torch.float32:
        _need(o, "o", q.dtype)
    else:
        _need_rows(o, "o", o)
        if tuple(o.shape) != tuple(q.shape) or o.dtype != q.dtype:
            raise ValueError("o must match q's shape and dtype")
    _need(lse, "lse", torch.float32)
    desc, keep = _desc(q, b, head_classes, scale, o)
    st = csr.struct()
    _check("gsa_attn_fwd", library().gsa_attn_fwd(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(st), ctypes.byref(desc),
                                                  _ptr(o), _ptr(lse), _stream(stream)))
    del keep
    return o, lse


def gsa_attn_bwd_workspace(q: torch.Tensor, b: int, head_classes) -> int:
    desc, keep = _desc(q, b, head_classes, 0.0)
    return int(library().gsa_attn_bwd_workspace(ctypes.byref(desc)))


def gsa_attn_bwd(q, k, v, o, lse, do, csr: BlockCsr, head_classes, b: int, scale: float = 0.0,
                 dq=None, dk=None, dv=None, workspace: torch.Tensor | None = None, stream=None):
    """Gradients (dq, dk, dv) of gsa_attn_fwd for upstream gradient do.
    Strided views as in gsa_attn_fwd: k, v, dq, dk, dv with q's strides, do
    with o's; dq, dk, dv default to q's strides when q is dense, else they
    must be given."""
    if dq is None or dk is None or dv is None:
        if not q.is_contiguous():
            raise ValueError("pass dq, dk and dv (with q's strides) for a strided q")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t in (("q", q), ("k", k), ("v", v), ("dq", dq), ("dk", dk), ("dv", dv)):
        _need_rows(t, name, q)
    _need_rows(o, "o", o)
    _need_rows(do, "do", o)
    if tuple(o.shape) != tuple(q.shape):
        raise ValueError("o must match q's shape")
    _need(lse, "lse", torch.float32, 3)
    if len(head_classes) != q.shape[1]:
        raise ValueError("one head class per head")
    desc, keep = _desc(q, b, head_classes, scale, o)
    need = int(library().gsa_attn_bwd_workspace(ctypes.byref(desc)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace")
    st = csr.struct()
    _check("gsa_attn_bwd", library().gsa_attn_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), ctypes.byref(st), ctypes.byref(desc),
        _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    del keep
    return dq, dk, dv


def gsa_attn_bwd_noalloc_max_rows() -> int:
    """Query rows (B·H·L) the built-in scratch of gsa_attn_bwd_noalloc holds."""
    fn = library().gsa_attn_bwd_noalloc_max_rows
    fn.argtypes = []
    fn.restype = ctypes.c_int64
    return int(fn())


def gsa_attn_bwd_noalloc(q, k, v, o, lse, do, csr: BlockCsr, head_classes, b: int, scale: float = 0.0,
                         dq=None, dk=None, dv=None, stream=None):
    """gsa_attn_bwd without a workspace argument: the library's built-in
    scratch array is used and nothing is allocated by the library (for
    callers that cannot allocate device memory).  Calls that overlap on the
    GPU race on that array; the first call on a device must precede any
    stream capture."""
    lib = library()
    fn = lib.gsa_attn_bwd_noalloc
    vp = ctypes.c_void_p
    fn.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.POINTER(_Csr), ctypes.POINTER(_AttnDesc), vp, vp, vp, vp]
    fn.restype = ctypes.c_int
    if dq is None or dk is None or dv is None:
        if not q.is_contiguous():
            raise ValueError("pass dq, dk and dv (with q's strides) for a strided q")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t in (("q", q), ("k", k), ("v", v), ("dq", dq), ("dk", dk), ("dv", dv)):
        _need_rows(t, name, q)
    _need_rows(o, "o", o)
    _need_rows(do, "do", o)
    _need(lse, "lse", torch.float32, 3)
    desc, keep = _desc(q, b, head_classes, scale, o)
    st = csr.struct()
    _check("gsa_attn_bwd_noalloc", fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), ctypes.byref(st),
                                      ctypes.byref(desc), _ptr(dq), _ptr(dk), _ptr(dv), _stream(stream)))
    del keep
    return dq, dk, dv


# ------------------------------------------------------------ ByteLM block

LM_WEIGHTS = ("emb", "ln1_g", "ln1_b", "w_qkv", "w_o", "ln2_g", "ln2_b", "w_1", "w_2")
_LM_F32 = ("ln1_g", "ln1_b", "ln2_g", "ln2_b")


class _LmDesc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("L", ctypes.c_int32), ("D", ctypes.c_int32), ("H", ctypes.c_int32),
        ("F", ctypes.c_int32), ("b", ctypes.c_int32), ("head_classes", ctypes.c_void_p),
        ("ln_eps", ctypes.c_float),
    ]


class _LmPtrs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in LM_WEIGHTS]


def _lm_fns():
    lib = library()
    vp = ctypes.c_void_p
    lib.gsa_lm_block_workspace.argtypes = [ctypes.POINTER(_LmDesc)]
    lib.gsa_lm_block_workspace.restype = ctypes.c_size_t
    lib.gsa_lm_block_fwd.argtypes = [vp, ctypes.POINTER(_LmPtrs), ctypes.POINTER(_Csr), ctypes.POINTER(_LmDesc),
                                     vp, vp, ctypes.c_size_t, vp]
    lib.gsa_lm_block_fwd.restype = ctypes.c_int
    lib.gsa_lm_block_bwd.argtypes = [vp, ctypes.POINTER(_LmPtrs), ctypes.POINTER(_Csr), ctypes.POINTER(_LmDesc),
                                     vp, ctypes.POINTER(_LmPtrs), vp, ctypes.c_size_t, vp]
    lib.gsa_lm_block_bwd.restype = ctypes.c_int
    i32, i64 = ctypes.c_int32, ctypes.c_int64
    lib.gsa_lm_gemm.argtypes = [i32, i32, i32, i32, i32, vp, i64, vp, i64, ctypes.c_float, vp, i64, vp, i64, i32,
                                i32, vp, i64, vp, ctypes.c_size_t, vp]
    lib.gsa_lm_gemm.restype = ctypes.c_int
    lib.gsa_lm_gemm_workspace.argtypes = [i32, i32, i32, i32]
    lib.gsa_lm_gemm_workspace.restype = ctypes.c_size_t
    return lib


GEMM_EPI_NONE, GEMM_EPI_GELU_AUX, GEMM_EPI_DGELU = 0, 1, 2


def gsa_lm_gemm_workspace(M: int, N: int, K: int, out32: bool) -> int:
    """Scratch bytes gsa_lm_gemm needs for an M x N product over K (0 unless a float32 product splits K)."""
    return int(_lm_fns().gsa_lm_gemm_workspace(int(M), int(N), int(K), int(out32)))


def gsa_lm_gemm(a: torch.Tensor, b: torch.Tensor, ta: bool = False, tb: bool = False, c: torch.Tensor | None = None,
                beta: float = 0.0, out32: bool = False, epi: int = GEMM_EPI_NONE, aux: torch.Tensor | None = None,
                d: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Row-major D = op(A) op(B) (+ beta C, or a GELU epilogue) on the
    library's tcgen05 GEMM.  ta: a is [K, M] (else [M, K]); tb: b is [N, K]
    (else [K, N]).  bf16 operands; D bf16, or float32 with out32.  epi
    GEMM_EPI_GELU_AUX writes GELU(acc) to D and acc to aux; GEMM_EPI_DGELU
    returns acc * GELU'(aux)."""
    lib = _lm_fns()
    _need(a, "a", torch.bfloat16, 2)
    _need(b, "b", torch.bfloat16, 2)
    M = a.shape[1] if ta else a.shape[0]
    K = a.shape[0] if ta else a.shape[1]
    N = b.shape[0] if tb else b.shape[1]
    if (b.shape[1] if tb else b.shape[0]) != K:
        raise ValueError("inner dimensions differ")
    if d is None:
        d = torch.empty((M, N), dtype=torch.float32 if out32 else torch.bfloat16, device=a.device)
    ws_bytes = gsa_lm_gemm_workspace(M, N, K, out32)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=a.device)
    if epi == GEMM_EPI_GELU_AUX and aux is None:
        aux = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    _check("gsa_lm_gemm", lib.gsa_lm_gemm(int(ta), int(tb), M, N, K, _ptr(a), a.stride(0), _ptr(b), b.stride(0),
                                          float(beta), _ptr(c) if c is not None else None,
                                          c.stride(0) if c is not None else 0, _ptr(d), d.stride(0), int(out32),
                                          int(epi), _ptr(aux) if aux is not None else None,
                                          aux.stride(0) if aux is not None else 0, _ptr(ws), ws_bytes,
                                          _stream(stream)))
    return d


def _lm_desc(B, L, D, H, F, head_classes, b, eps):
    hc = (ctypes.c_uint8 * H)(*[int(c) for c in head_classes])
    return _LmDesc(B, L, D, H, F, int(b), ctypes.cast(hc, ctypes.c_void_p), float(eps)), hc


def _lm_weights(w: dict):
    """(D, H, F) of a weight dict, checking dtypes and shapes."""
    D = w["emb"].shape[1]
    F = w["w_1"].shape[0]
    shapes = {"emb": (256, D), "w_qkv": (3 * D, D), "w_o": (D, D), "w_1": (F, D), "w_2": (D, F)}
    for n in LM_WEIGHTS:
        _need(w[n], n, torch.float32 if n in _LM_F32 else torch.bfloat16)
        if tuple(w[n].shape) != shapes.get(n, (D,)):
            raise ValueError(f"{n} must have shape {shapes.get(n, (D,))}")
    return D, D // 64, F


def gsa_lm_block_workspace(B: int, L: int, D: int, H: int, F: int, head_classes, b: int = 64,
                           eps: float = 1e-5) -> int:
    desc, keep = _lm_desc(B, L, D, H, F, head_classes, b, eps)
    return int(_lm_fns().gsa_lm_block_workspace(ctypes.byref(desc)))


def gsa_lm_block_fwd(data: torch.Tensor, weights: dict, csr: BlockCsr, head_classes, b: int = 64,
                     eps: float = 1e-5, y: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                     stream=None):
    """One ByteLM block forward over bytes data [B, L] (uint8): returns
    (y [B, L, D] bf16, workspace).  Pass the returned workspace to
    gsa_lm_block_bwd."""
    _need(data, "data", torch.uint8, 2)
    B, L = data.shape
    D, H, F = _lm_weights(weights)
    lib = _lm_fns()
    desc, keep = _lm_desc(B, L, D, H, F, head_classes, b, eps)
    need = int(lib.gsa_lm_block_workspace(ctypes.byref(desc)))
    if need == 0:
        raise ValueError("invalid ByteLM block shape")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=data.device)
    if y is None:
        y = torch.empty((B, L, D), dtype=torch.bfloat16, device=data.device)
    _need(y, "y", torch.bfloat16)
    _need(workspace, "workspace")
    wp = _LmPtrs(*[weights[n].data_ptr() for n in LM_WEIGHTS])
    st = csr.struct()
    _check("gsa_lm_block_fwd", lib.gsa_lm_block_fwd(_ptr(data), ctypes.byref(wp), ctypes.byref(st),
                                                    ctypes.byref(desc), _ptr(y), _ptr(workspace),
                                                    workspace.numel(), _stream(stream)))
    del keep
    return y, workspace


def gsa_lm_block_bwd(data: torch.Tensor, weights: dict, csr: BlockCsr, head_classes, dy: torch.Tensor,
                     workspace: torch.Tensor, b: int = 64, eps: float = 1e-5, grads: dict | None = None,
                     stream=None) -> dict:
    """Gradients (float32, one per weight) of <y, dy> for the forward that
    last used this workspace."""
    _need(data, "data", torch.uint8, 2)
    B, L = data.shape
    D, H, F = _lm_weights(weights)
    _need(dy, "dy", torch.bfloat16, 3)
    if tuple(dy.shape) != (B, L, D):
        raise ValueError("dy must be [B, L, D]")
    _need(workspace, "workspace")
    if grads is None:
        grads = {n: torch.empty(weights[n].shape, dtype=torch.float32, device=data.device) for n in LM_WEIGHTS}
    for n in LM_WEIGHTS:
        _need(grads[n], "grad " + n, torch.float32)
    lib = _lm_fns()
    desc, keep = _lm_desc(B, L, D, H, F, head_classes, b, eps)
    wp = _LmPtrs(*[weights[n].data_ptr() for n in LM_WEIGHTS])
    gp = _LmPtrs(*[grads[n].data_ptr() for n in LM_WEIGHTS])
    st = csr.struct()
    _check("gsa_lm_block_bwd", lib.gsa_lm_block_bwd(_ptr(data), ctypes.byref(wp), ctypes.byref(st),
                                                    ctypes.byref(desc), _ptr(dy), ctypes.byref(gp),
                                                    _ptr(workspace), workspace.numel(), _stream(stream)))
    del keep
    return grads


def gsa_device_error(clear: bool = True) -> int:
    """The library's device error word (0 = no kernel gave up a wait)."""
    code = ctypes.c_int32(0)
    library().gsa_device_error(ctypes.byref(code), 1 if clear else 0)
    return int(code.value)
