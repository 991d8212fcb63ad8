"""Strided tensor layouts (gsa_attn_layout): Q, K, V read from one
token-major [B, L, 3, H, d] projection output, O and dO as [B, L, H, d] rows,
dQ, dK, dV written into a [B, L, 3, H, d] buffer.  The kernels are the same,
only the addresses differ, so every output must equal the dense-layout run
bit for bit (which the other attention tests pin to the oracle)."""
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gsa():
    from content_adaptive_block_b200 import build
    build.build()
    import content_adaptive_block_b200 as g
    return g


@pytest.mark.parametrize("B,L,H,d,w", [(8, 8192, 12, 64, 2), (2, 4096, 4, 128, 3), (3, 17 * 64, 2, 64, 1)])
def test_token_major_layout_matches_dense(gsa, B, L, H, d, w):
    g = torch.Generator(device="cuda")
    g.manual_seed(B * 1000 + L + d)
    qkv = torch.randn((B, L, 3, H, d), generator=g, device="cuda").bfloat16()
    dob = torch.randn((B, L, H, d), generator=g, device="cuda").bfloat16()
    q, k, v = (qkv[:, :, i].permute(0, 2, 1, 3) for i in range(3))   # [B, H, L, d] views
    do = dob.permute(0, 2, 1, 3)
    hc = [(0, 1, 2)[h % 3] for h in range(H)]
    x = torch.from_numpy(W.custom_bytes(B, L, ("uniform", 0.2, 0.6), seed=L + H)).cuda()
    _, _, csr = gsa.gsa_mask_pipeline(x, 64, w) if L // 64 <= 1024 else (None, None, None)

    # dense run
    qc, kc, vc, doc = (t.contiguous() for t in (q, k, v, do))
    o_ref, lse_ref = gsa.gsa_attn_fwd(qc, kc, vc, csr, hc, 64)
    dq_ref, dk_ref, dv_ref = gsa.gsa_attn_bwd(qc, kc, vc, o_ref, lse_ref, doc, csr, hc, 64)

    # strided run
    obuf = torch.empty((B, L, H, d), dtype=torch.bfloat16, device="cuda")
    o = obuf.permute(0, 2, 1, 3)
    o2, lse = gsa.gsa_attn_fwd(q, k, v, csr, hc, 64, o=o)
    dbuf = torch.empty((B, L, 3, H, d), dtype=torch.bfloat16, device="cuda")
    dq, dk, dv = (dbuf[:, :, i].permute(0, 2, 1, 3) for i in range(3))
    gsa.gsa_attn_bwd(q, k, v, o, lse, do, csr, hc, 64, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    assert o2.data_ptr() == obuf.data_ptr()
    assert torch.equal(o, o_ref)
    assert torch.equal(lse, lse_ref)
    assert torch.equal(dq, dq_ref)
    assert torch.equal(dk, dk_ref)
    assert torch.equal(dv, dv_ref)
