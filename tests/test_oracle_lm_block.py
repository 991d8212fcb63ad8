"""The oracle's ByteLM block against facts that do not come from it: torch's
own layer_norm and tanh-GELU, the pinned block-sparse attention oracle,
central finite differences of the whole block, the dense form against the
sampled-rows form, closed-form special cases (zero output projections leave
the embedding; a diagonal-only mask returns V), and the parameter count."""
import math

import numpy as np
import torch

from oracle import attention as oatt
from oracle import lm_block as olm
from oracle import mask as om


def _weights(D, F, seed, scale=0.2):
    rng = np.random.default_rng(seed)
    return {
        "emb": rng.normal(0, 1, (256, D)), "ln1_g": 1 + 0.1 * rng.normal(size=D), "ln1_b": 0.1 * rng.normal(size=D),
        "ln2_g": 1 + 0.1 * rng.normal(size=D), "ln2_b": 0.1 * rng.normal(size=D),
        "w_qkv": scale * rng.normal(size=(3 * D, D)), "w_o": scale * rng.normal(size=(D, D)),
        "w_1": scale * rng.normal(size=(F, D)), "w_2": scale * rng.normal(size=(D, F)),
    }


def _masks(bytes_, b, w, H, classes):
    from oracle import flags as ofl
    from oracle import deflate1
    S, L = bytes_.shape
    ln = deflate1.block_lengths(bytes_, b)
    fl = ofl.literal_flags(ln, b)
    bm = [[om.block_mask(fl[s], w, classes[h]) for h in range(H)] for s in range(S)]
    tm = [[torch.from_numpy(om.token_mask(bm[s][h], b)) for h in range(H)] for s in range(S)]
    return bm, tm


def test_layer_norm_matches_torch():
    x = torch.randn(5, 24, dtype=torch.float64)
    g, b = torch.randn(24, dtype=torch.float64), torch.randn(24, dtype=torch.float64)
    assert torch.allclose(olm.layer_norm(x, g, b), torch.nn.functional.layer_norm(x, (24,), g, b, 1e-5),
                          atol=1e-12)


def test_gelu_matches_torch_tanh_form():
    u = torch.linspace(-8, 8, 1001, dtype=torch.float64)
    assert torch.allclose(olm.gelu_tanh(u), torch.nn.functional.gelu(u, approximate="tanh"), atol=1e-14)


def test_masked_attention_matches_the_block_sparse_oracle():
    rng = np.random.default_rng(1)
    n, b, d = 6, 8, 16
    fl = np.array([1, 0, 1, 1, 0, 1], dtype=np.uint8)
    m = om.block_mask(fl, 1, om.HYBRID)
    q, k, v = (rng.normal(size=(n * b, d)) for _ in range(3))
    want, _ = oatt.forward(q, k, v, m, b)
    got = olm.masked_attention(*(torch.from_numpy(x) for x in (q, k, v)), torch.from_numpy(om.token_mask(m, b)))
    assert np.abs(got.numpy() - want).max() < 1e-12


def test_zero_projections_leave_the_embedding():
    rng = np.random.default_rng(2)
    D, F, H = 16, 32, 2
    w = _weights(D, F, 3)
    w["w_o"][:] = 0
    w["w_2"][:] = 0
    x = rng.integers(0, 256, size=(2, 32), dtype=np.uint8)
    _, tm = _masks(x, 8, 1, H, [0, 2])
    y = olm.block_forward(x, {k: torch.from_numpy(v) for k, v in w.items()}, tm, H).numpy()
    assert np.array_equal(y, w["emb"][x.astype(np.int64)])


def test_diagonal_mask_returns_v():
    # each token sees only itself: the attention output is its own V row
    D, H, F, L = 16, 2, 32, 12
    w = _weights(D, F, 4)
    x = np.arange(L, dtype=np.uint8)[None, :]
    eye = torch.eye(L, dtype=torch.bool)
    wt = {k: torch.from_numpy(v) for k, v in w.items()}
    h = olm.layer_norm(wt["emb"][torch.from_numpy(x.astype(np.int64))], wt["ln1_g"], wt["ln1_b"])
    v = h @ wt["w_qkv"][2 * D:].T
    x1 = wt["emb"][torch.from_numpy(x.astype(np.int64))] + v @ wt["w_o"].T
    want = x1 + olm.gelu_tanh(olm.layer_norm(x1, wt["ln2_g"], wt["ln2_b"]) @ wt["w_1"].T) @ wt["w_2"].T
    got = olm.block_forward(x, wt, [[eye, eye]], H)
    assert torch.allclose(got, want, atol=1e-12)


def test_rows_form_matches_dense_form():
    rng = np.random.default_rng(5)
    D, H, F, b = 32, 2, 64, 8
    classes = [1, 2]
    x = rng.integers(0, 256, size=(1, 10 * b), dtype=np.uint8)
    x[0, 3 * b:5 * b] = 97   # compressible blocks next to random ones
    w = _weights(D, F, 6)
    bm, tm = _masks(x, b, 1, H, classes)
    y = olm.block_forward(x, {k: torch.from_numpy(v) for k, v in w.items()}, tm, H).numpy()
    qb = [0, 4, 9]
    rows, yr = olm.block_rows_forward(x[0], w, bm[0], H, b, qb)
    assert np.abs(yr - y[0, rows]).max() < 1e-10


def test_backward_matches_finite_differences():
    rng = np.random.default_rng(7)
    D, H, F, b = 8, 2, 16, 4
    x = rng.integers(0, 256, size=(2, 4 * b), dtype=np.uint8)
    w = _weights(D, F, 8, scale=0.5)
    _, tm = _masks(x, b, 1, H, [0, 2])
    dy = rng.normal(size=(2, 4 * b, D))
    _, grads = olm.block_forward_backward(x, w, tm, H, dy)

    def f(wd):
        y = olm.block_forward(x, {k: torch.from_numpy(v) for k, v in wd.items()}, tm, H).numpy()
        return float((y * dy).sum())

    eps = 1e-6
    for name in w:
        flat = w[name].reshape(-1)
        idx = rng.choice(flat.size, size=min(4, flat.size), replace=False)
        if name == "emb":
            idx = np.array([int(x[0, 0]) * D, int(x[1, 3]) * D + 2])   # rows that are used
        for i in idx:
            wp = {k: v.copy() for k, v in w.items()}
            wm = {k: v.copy() for k, v in w.items()}
            wp[name].reshape(-1)[i] += eps
            wm[name].reshape(-1)[i] -= eps
            fd = (f(wp) - f(wm)) / (2 * eps)
            assert abs(fd - grads[name].reshape(-1)[i]) <= 1e-6 * max(1.0, abs(fd)), (name, i)


def test_parameter_count():
    # 12 blocks of width 768 (MLP 3072) hold ~85M weights, the paper's 92M size class
    per_block = olm.parameter_count(768, 3072) - 256 * 768
    assert per_block == 4 * 768 + 4 * 768 * 768 + 2 * 768 * 3072
    assert 84e6 < 12 * per_block < 86e6
    assert math.isclose(12 * (4 * 768 ** 2 + 2 * 768 * 3072) / 1e6, 84.93, rel_tol=1e-3)
