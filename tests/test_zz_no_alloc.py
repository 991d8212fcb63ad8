"""gsa_attn_bwd_noalloc: the backward for callers that cannot allocate device
memory (a host framework that owns every device byte, or a loop that cannot
pay for cudaMalloc's synchronisation).  Its scratch is a fixed array inside
the library, so the caller passes no workspace.

Checked through the C ABI against gsa_attn_bwd (which takes a caller-made
workspace) on two calls in a row, within the backward's tolerance (relative
L2 <= 2e-2 per gradient); bit for bit over calls whose shapes change in
between (the array is shared and never cleared); plus the host-side size
limit.  This file is
collected last so a run that stops at the first failure has run the rest."""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

TOL_REL_L2 = 2e-2


@pytest.fixture(scope="module")
def gsa():
    from content_adaptive_block_b200 import build
    build.build()
    import content_adaptive_block_b200 as g
    return g


def _noalloc_fn(lib, gsa):
    fn = lib.gsa_attn_bwd_noalloc
    vp = ctypes.c_void_p
    fn.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.POINTER(gsa._Csr), ctypes.POINTER(gsa._AttnDesc), vp, vp, vp, vp]
    fn.restype = ctypes.c_int
    return fn


def _rel(a, b):
    a = a.float()
    b = b.float()
    return float(torch.linalg.norm(a - b) / torch.linalg.norm(b))


@pytest.mark.parametrize("d", [64, 128])
def test_noalloc_matches_workspace_backward(gsa, d):
    lib = gsa.library()
    fn = _noalloc_fn(lib, gsa)
    S, H, n, b, w = 2, 4, 9, 64, 1
    hc = [0, 1, 2, 2]
    rng = np.random.default_rng(d)
    fl = torch.from_numpy((rng.random((S, n)) < 0.5).astype(np.uint8)).cuda()
    csr = gsa.gsa_build_block_csr(fl, w)
    q, k, v, do = (t.cuda() for t in W.random_tensors((S, H, n * b, d), 4, torch.bfloat16, seed=31 + d))
    o, lse = gsa.gsa_attn_fwd(q, k, v, csr, hc, b)
    ref = gsa.gsa_attn_bwd(q, k, v, o, lse, do, csr, hc, b)

    hcs = (ctypes.c_uint8 * H)(*hc)
    desc = gsa._AttnDesc(S, H, n * b, d, b, 1, 0.0, ctypes.cast(hcs, ctypes.c_void_p))
    st = csr.struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        dq, dk, dv = torch.full_like(q, float("nan")), torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))
        rc = fn(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
                ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(do.data_ptr()),
                ctypes.byref(st), ctypes.byref(desc), ctypes.c_void_p(dq.data_ptr()),
                ctypes.c_void_p(dk.data_ptr()), ctypes.c_void_p(dv.data_ptr()), stream)
        assert rc == 0, gsa.gsa_status_string(rc)
        torch.cuda.synchronize()
        assert gsa.gsa_device_error() == 0
        for got, want in zip((dq, dk, dv), ref):
            assert torch.isfinite(got.float()).all(), call
            assert _rel(got, want) <= TOL_REL_L2, call


def _call_noalloc(fn, gsa, q, k, v, o, lse, do, csr, hc, b):
    S, H, L, d = q.shape
    hcs = (ctypes.c_uint8 * H)(*hc)
    desc = gsa._AttnDesc(S, H, L, d, b, 1, 0.0, ctypes.cast(hcs, ctypes.c_void_p))
    st = csr.struct()
    dq, dk, dv = torch.full_like(q, float("nan")), torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))
    rc = fn(*(ctypes.c_void_p(t.data_ptr()) for t in (q, k, v, o, lse, do)), ctypes.byref(st), ctypes.byref(desc),
            *(ctypes.c_void_p(t.data_ptr()) for t in (dq, dk, dv)),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, gsa.gsa_status_string(rc)
    return dq, dk, dv


def test_noalloc_shape_changes_between_calls(gsa):
    """The shared array keeps the last call's contents and its regions sit at
    offsets that depend on B*H*L: a large call, a smaller one, then the large
    one again must each give gsa_attn_bwd's gradients (with a fresh workspace)
    bit for bit, since both run the same deterministic kernels."""
    lib = gsa.library()
    fn = _noalloc_fn(lib, gsa)
    b = 64
    shapes = [(2, 4, 9, 64, 1), (1, 3, 5, 64, 2), (2, 4, 9, 64, 1), (1, 2, 7, 128, 1)]
    for i, (S, H, n, d, w) in enumerate(shapes):
        hc = [(0, 1, 2, 2)[h % 4] for h in range(H)]
        rng = np.random.default_rng(100 + i)
        fl = torch.from_numpy((rng.random((S, n)) < 0.5).astype(np.uint8)).cuda()
        csr = gsa.gsa_build_block_csr(fl, w)
        q, k, v, do = (t.cuda() for t in W.random_tensors((S, H, n * b, d), 4, torch.bfloat16, seed=200 + i))
        o, lse = gsa.gsa_attn_fwd(q, k, v, csr, hc, b)
        ref = gsa.gsa_attn_bwd(q, k, v, o, lse, do, csr, hc, b)
        got = _call_noalloc(fn, gsa, q, k, v, o, lse, do, csr, hc, b)
        torch.cuda.synchronize()
        assert gsa.gsa_device_error() == 0
        for name, g_, r_ in zip(("dq", "dk", "dv"), got, ref):
            assert torch.equal(g_, r_), (i, name)


def test_noalloc_rejects_rows_beyond_its_scratch(gsa):
    lib = gsa.library()
    fn = _noalloc_fn(lib, gsa)
    lib.gsa_attn_bwd_noalloc_max_rows.restype = ctypes.c_int64
    max_rows = int(lib.gsa_attn_bwd_noalloc_max_rows())
    assert max_rows == 1 << 21
    # B*H*L one block above the limit (checked on the host, nothing runs)
    n, b, H = 2048, 64, 17
    S = 1
    assert S * H * n * b > max_rows
    hcs = (ctypes.c_uint8 * H)(*([0] * H))
    desc = gsa._AttnDesc(S, H, n * b, 64, b, 1, 0.0, ctypes.cast(hcs, ctypes.c_void_p))
    fake = 0x1000
    st = gsa._Csr(S, n, 1, 7, gsa.gsa_csr_capacity(n), fake, fake, fake, fake, fake, fake)
    p = ctypes.c_void_p(fake)
    rc = fn(p, p, p, p, p, p, ctypes.byref(st), ctypes.byref(desc), p, p, p, ctypes.c_void_p(0))
    assert rc == 3   # GSA_ERR_CAPACITY
