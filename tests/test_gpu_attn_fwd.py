"""GPU parity of the attention forward against the float64 oracle.

Tolerances (max-abs over outputs): 1e-5 for the float32 CUDA-core path,
2e-2 for the bf16 tensor-core path with unit-variance V (the oracle runs in
float64 on the same bf16-rounded inputs).  LSE (float32 on both paths) is
compared to 1e-3 absolute for bf16 inputs, 1e-5 for float32."""
import numpy as np
import pytest
import torch

import workloads as W
from parity_sampling import class_pairs
from oracle import attention as oatt, deflate1, flags as oflags, mask as omask

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 2e-2
TOL_LSE_BF16 = 1e-3


@pytest.fixture(scope="module")
def gsa():
    from content_adaptive_block_b200 import build
    build.build()
    import content_adaptive_block_b200 as g
    return g


def _flags_for(x: np.ndarray, b: int) -> np.ndarray:
    return oflags.literal_flags(deflate1.block_lengths(x, b, nthreads=8), b)


def _run_fwd(gsa, q, k, v, fl, w, hc, b):
    csr = gsa.gsa_build_block_csr(torch.from_numpy(fl.astype(np.uint8)).cuda(), w)
    o, lse = gsa.gsa_attn_fwd(q.cuda(), k.cuda(), v.cuda(), csr, list(hc), b)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    return o.float().cpu().numpy(), lse.cpu().numpy()


def _compare(o, lse, q, k, v, fl, w, hc, b, tol_o, tol_l, pairs=None, q_blocks=None):
    S, H = q.shape[:2]
    worst = 0.0
    for s in range(S):
        for h in range(H):
            if pairs is not None and (s, h) not in pairs:
                continue
            m = omask.block_mask(fl[s], w, int(hc[h]))
            ro, rl = oatt.forward(q[s, h].float(), k[s, h].float(), v[s, h].float(), m, b, q_blocks=q_blocks)
            sel = ~np.isnan(rl)
            err = np.abs(o[s, h][sel] - ro[sel]).max()
            lerr = np.abs(lse[s, h][sel] - rl[sel]).max()
            worst = max(worst, err)
            assert err <= tol_o, (s, h, err)
            assert lerr <= tol_l, (s, h, lerr)
    return worst


def test_tiny_fp32_config(gsa):
    wl = W.WORKLOADS["tiny_fp32"]
    x = W.batch_bytes(wl)
    fl = _flags_for(x, wl.b)
    q, k, v = W.qkv(wl, seed=0)
    o, lse = _run_fwd(gsa, q, k, v, fl, wl.w, wl.head_classes(), wl.b)
    _compare(o, lse, q, k, v, fl, wl.w, wl.head_classes(), wl.b, TOL_F32, TOL_F32)


@pytest.mark.parametrize("b,d", [(16, 16), (32, 64), (64, 128), (7, 32)])
def test_fp32_other_shapes(gsa, b, d):
    S, H, n = 2, 3, 5
    rng = np.random.default_rng(b * d)
    fl = (rng.random((S, n)) < 0.5).astype(np.uint8)
    q, k, v = W.random_tensors((S, H, n * b, d), 3, torch.float32, seed=b + d)
    hc = np.array([0, 1, 2], dtype=np.uint8)
    o, lse = _run_fwd(gsa, q, k, v, fl, 1, hc, b)
    _compare(o, lse, q, k, v, fl, 1, hc, b, TOL_F32, TOL_F32)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n,w", [(1, 1), (2, 0), (3, 1), (9, 2), (16, 2), (33, 4)])
def test_bf16_small_shapes(gsa, d, n, w):
    # several 128-row tiles, an odd block count (a half-empty last tile), all classes
    S, H, b = 2, 4, 64
    rng = np.random.default_rng(n * 10 + w + d)
    fl = (rng.random((S, n)) < 0.45).astype(np.uint8)
    hc = np.array([0, 1, 2, 2], dtype=np.uint8)
    q, k, v = W.random_tensors((S, H, n * b, d), 3, torch.bfloat16, seed=n + d)
    o, lse = _run_fwd(gsa, q, k, v, fl, w, hc, b)
    _compare(o, lse, q, k, v, fl, w, hc, b, TOL_BF16, TOL_LSE_BF16)


@pytest.mark.parametrize("d", [64, 128])
def test_bf16_special_masks(gsa, d):
    S, H, n, b = 3, 3, 12, 64
    fl = np.stack([np.ones(n), np.zeros(n), (np.arange(n) % 3 == 0)]).astype(np.uint8)
    hc = np.array([0, 1, 2], dtype=np.uint8)
    q, k, v = W.random_tensors((S, H, n * b, d), 3, torch.bfloat16, seed=7 + d)
    for w in (0, 2, n):
        o, lse = _run_fwd(gsa, q, k, v, fl, w, hc, b)
        _compare(o, lse, q, k, v, fl, w, hc, b, TOL_BF16, TOL_LSE_BF16)


def test_bf16_large_scores(gsa):
    # scaled-up queries make the running max jump between tiles (O rescaling)
    S, H, n, b, d = 1, 3, 20, 64, 64
    fl = (np.arange(n)[None, :] % 2 == 0).astype(np.uint8)
    hc = np.array([0, 1, 2], dtype=np.uint8)
    q, k, v = W.random_tensors((S, H, n * b, d), 3, torch.float32, seed=3)
    ramp = torch.linspace(0.2, 4.0, n * b)[None, None, :, None]
    q = (q * 3.0).to(torch.bfloat16)
    k = (k * ramp).to(torch.bfloat16)
    v = v.to(torch.bfloat16)
    o, lse = _run_fwd(gsa, q, k, v, fl, 1, hc, b)
    _compare(o, lse, q, k, v, fl, 1, hc, b, TOL_BF16, 5e-3)


def test_b8_4k_full(gsa):
    wl = W.WORKLOADS["b8_4k"]
    x = W.batch_bytes(wl)
    fl = _flags_for(x, wl.b)
    q, k, v = W.qkv(wl, seed=0)
    o, lse = _run_fwd(gsa, q, k, v, fl, wl.w, wl.head_classes(), wl.b)
    _compare(o, lse, q, k, v, fl, wl.w, wl.head_classes(), wl.b, TOL_BF16, TOL_LSE_BF16)


def test_b8_8k_sampled(gsa):
    wl = W.WORKLOADS["b8_8k"]
    x = W.batch_bytes(wl)
    fl = _flags_for(x, wl.b)
    q, k, v = W.qkv(wl, seed=0)
    o, lse = _run_fwd(gsa, q, k, v, fl, wl.w, wl.head_classes(), wl.b)
    hc = wl.head_classes()
    pairs = class_pairs(wl.S, hc, 4, seed=0)   # 4 distinct (sample, head) per class
    assert len(pairs) == 12
    _compare(o, lse, q, k, v, fl, wl.w, hc, wl.b, TOL_BF16, TOL_LSE_BF16, pairs=pairs)


def test_b1_64k_sampled(gsa):
    wl = W.WORKLOADS["b1_64k"]
    x = W.batch_bytes(wl)
    fl = _flags_for(x, wl.b)
    q, k, v = W.qkv(wl, seed=0)
    o, lse = _run_fwd(gsa, q, k, v, fl, wl.w, wl.head_classes(), wl.b)
    hc = wl.head_classes()
    lit = np.nonzero(fl[0])[0]
    qb = sorted(set([0, 1, wl.N - 1, int(lit[-1]), int(lit[len(lit) // 2])] +
                    np.random.default_rng(1).integers(0, wl.N, 12).tolist()))
    pairs = class_pairs(wl.S, hc, 4, seed=1)   # 4 distinct heads per class (the one sample)
    assert len(pairs) == 12
    _compare(o, lse, q, k, v, fl, wl.w, hc, wl.b, TOL_BF16, TOL_LSE_BF16, pairs=pairs, q_blocks=qb)


def test_bf16_concurrent_streams_and_counter_slots(gsa):
    """The d=64 bf16 forward's persistent CTAs draw items from a device-global
    counter slot per call: four calls in flight on four streams, and more calls
    in a row than there are slots, give the outputs of one call at a time,
    bit for bit (each item's arithmetic does not depend on the CTA taking it)."""
    wl = W.WORKLOADS["b8_4k"]
    fl = _flags_for(W.batch_bytes(wl), wl.b)
    hc = list(wl.head_classes())
    csr = gsa.gsa_build_block_csr(torch.from_numpy(fl.astype(np.uint8)).cuda(), wl.w)
    ins = [[t.cuda() for t in W.qkv(wl, seed=seed)] for seed in range(4)]
    want = []
    for q, k, v in ins:
        o, lse = gsa.gsa_attn_fwd(q, k, v, csr, hc, wl.b)
        want.append((o.clone(), lse.clone()))
    torch.cuda.synchronize()
    outs = [(torch.empty_like(q), torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)) for q, _, _ in ins]
    streams = [torch.cuda.Stream() for _ in ins]
    for (q, k, v), (o, lse), st in zip(ins, outs, streams):
        st.wait_stream(torch.cuda.current_stream())
        gsa.gsa_attn_fwd(q, k, v, csr, hc, wl.b, o=o, lse=lse, stream=st)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    for (o, lse), (wo, wlse) in zip(outs, want):
        assert torch.equal(o, wo) and torch.equal(lse, wlse)
    # more calls than counter slots (256): every slot comes back to zero
    q, k, v = ins[0]
    o, lse = outs[0]
    for _ in range(300):
        gsa.gsa_attn_fwd(q, k, v, csr, hc, wl.b, o=o, lse=lse)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    assert torch.equal(o, want[0][0]) and torch.equal(lse, want[0][1])
