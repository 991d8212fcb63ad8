"""The ByteLM block's GEMM (gsa_lm_gemm: tcgen05 tensor cores, TMA, TMEM)
against a float32 reference of the same bf16 operands: every operand
storage order, a row count that ends inside a 128-row tile, the residual
add, the GELU epilogues (tanh form, as the block's oracle), float32 output
with and without a K split, and bit-for-bit repeatability.

Bars: relative L2 <= 1e-2 for bf16 outputs (one bf16 rounding of the
result; the reference rounds nothing), <= 1e-5 for float32 outputs (only
the summation order differs)."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gsa():
    from content_adaptive_block_b200 import build
    build.build()
    import content_adaptive_block_b200 as g
    return g


def _rel(a, b):
    return float(torch.linalg.norm(a.float() - b.float()) / torch.linalg.norm(b.float()))


def _ops(M, N, K, ta, tb, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    a = torch.randn((K, M) if ta else (M, K), generator=g, device="cuda").bfloat16()
    b = torch.randn((N, K) if tb else (K, N), generator=g, device="cuda").bfloat16()
    ref = (a.float().t() if ta else a.float()) @ (b.float().t() if tb else b.float())
    return a, b, ref


def _gelu(x):
    return 0.5 * x * (1 + torch.tanh(0.7978845608028654 * (x + 0.044715 * x ** 3)))


def _gelu_grad(x):
    t = torch.tanh(0.7978845608028654 * (x + 0.044715 * x ** 3))
    return 0.5 * (1 + t) + 0.5 * x * (1 - t * t) * 0.7978845608028654 * (1 + 3 * 0.044715 * x * x)


@pytest.mark.parametrize("ta,tb", [(False, True), (False, False), (True, True), (True, False)])
@pytest.mark.parametrize("M,N,K", [(256, 256, 64), (384, 512, 320), (200, 768, 768)])
def test_gemm_storage_orders(gsa, ta, tb, M, N, K):
    if ta and M % 128:
        pytest.skip("a [K][M] operand needs M in whole 128-row tiles")
    a, b, ref = _ops(M, N, K, ta, tb, seed=M + N + K + 2 * ta + tb)
    d = gsa.gsa_lm_gemm(a, b, ta=ta, tb=tb)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    assert _rel(d, ref) <= 1e-2, (ta, tb, M, N, K)


def test_gemm_residual_and_gelu_epilogues(gsa):
    M, N, K = 328, 512, 256
    a, b, ref = _ops(M, N, K, False, True, seed=7)
    c = torch.randn((M, N), device="cuda").bfloat16()
    d = gsa.gsa_lm_gemm(a, b, tb=True, c=c, beta=1.0)
    assert _rel(d, ref + c.float()) <= 1e-2
    aux = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    d = gsa.gsa_lm_gemm(a, b, tb=True, epi=gsa.GEMM_EPI_GELU_AUX, aux=aux)
    assert _rel(aux, ref) <= 1e-2
    assert _rel(d, _gelu(ref)) <= 1e-2
    d = gsa.gsa_lm_gemm(a, b, tb=True, epi=gsa.GEMM_EPI_DGELU, aux=aux)
    assert _rel(d, ref * _gelu_grad(aux.float())) <= 1e-2
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0


@pytest.mark.parametrize("M,N,K", [(256, 512, 4096), (768, 768, 8192)])
def test_gemm_float32_weight_gradient_shapes(gsa, M, N, K):
    # a [K][M] times [K][N]: the weight-gradient form; few tiles and long K split K
    a, b, ref = _ops(M, N, K, True, False, seed=K)
    assert gsa.gsa_lm_gemm_workspace(M, N, K, True) > 0
    d1 = gsa.gsa_lm_gemm(a, b, ta=True, out32=True)
    d2 = gsa.gsa_lm_gemm(a, b, ta=True, out32=True)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    assert d1.dtype == torch.float32
    assert _rel(d1, ref) <= 1e-5
    assert torch.equal(d1, d2)   # the split parts are summed in a fixed order


def test_gemm_rejects_unsupported_shapes(gsa):
    a = torch.zeros((128, 64), dtype=torch.bfloat16, device="cuda")
    b = torch.zeros((64, 200), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gsa.GsaError):
        gsa.gsa_lm_gemm(a, b)   # N not a multiple of 256
