"""ORACLE — test infrastructure only.  One ByteLM transformer block.

The pages train a byte-level language model ("ByteLM") with the adaptive
mask: Gzip-guided Sparse Attention (daiwk.github.io), fidelity line ("训练同参数
ByteLM") and section "论文离线与线上效果" (92M parameters, 8K bytes, 20K
steps); the arXiv abstract gives the same model size and context.  Neither
page states the block's layout.  Readings taken here (the plainest
transformer block of that size):
  * bytes index a learned embedding E [256, D]; no positional embedding
    (the causal mask orders the tokens);
  * pre-LayerNorm residual block: x1 = x0 + Attn(LN1(x0)) W_o^T,
    y = x1 + GELU(LN2(x1) W_1^T) W_2^T;
  * LayerNorm with gain and bias, biased variance, eps 1e-5;
  * linear layers without bias; W_qkv [3D, D] rows are (Q, K, V) x heads x 64;
  * GELU in its tanh form 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3)));
  * the attention is the block-sparse causal softmax attention of
    oracle.attention, softmax scale 1/sqrt(64), one head class per head;
  * D = 768, 12 heads of 64, F = 3072: 12 such blocks give ~85M weights,
    the size class of the paper's 92M model.
The backward is the chain rule of this forward, taken by torch autograd in
float64 from an upstream gradient dY.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from . import attention as oatt

LN_EPS = 1e-5


def layer_norm(x, g, b, eps=LN_EPS):
    """(x - mean) / sqrt(var + eps) * g + b over the last axis, biased variance."""
    mu = x.mean(dim=-1, keepdim=True)
    var = ((x - mu) ** 2).mean(dim=-1, keepdim=True)
    return (x - mu) / torch.sqrt(var + eps) * g + b


def gelu_tanh(u):
    return 0.5 * u * (1.0 + torch.tanh(math.sqrt(2.0 / math.pi) * (u + 0.044715 * u ** 3)))


def masked_attention(q, k, v, tmask):
    """q, k, v [T, 64] float64 tensors; tmask bool [T, T] token mask
    (oracle.mask.token_mask).  softmax(q k^T / sqrt(d), masked) v."""
    s = (q @ k.T) / math.sqrt(q.shape[1])
    s = s.masked_fill(~tmask, float("-inf"))
    return torch.softmax(s, dim=-1) @ v


def block_forward(bytes_, w: dict, masks, H: int):
    """bytes_ uint8 [S, L]; w: float64 tensors emb [256, D], ln1_g, ln1_b,
    ln2_g, ln2_b [D], w_qkv [3D, D], w_o [D, D], w_1 [F, D], w_2 [D, F];
    masks[s][h] bool [L, L] token mask of head h in sample s.
    Returns y [S, L, D] (float64, differentiable in w)."""
    S, L = bytes_.shape
    D = w["emb"].shape[1]
    dh = D // H
    idx = torch.as_tensor(np.asarray(bytes_, dtype=np.int64))
    x0 = w["emb"][idx]                                    # [S, L, D]
    h = layer_norm(x0, w["ln1_g"], w["ln1_b"])
    qkv = h @ w["w_qkv"].T                                # [S, L, 3D]
    outs = []
    for s in range(S):
        heads = []
        for hh in range(H):
            q = qkv[s, :, hh * dh:(hh + 1) * dh]
            k = qkv[s, :, D + hh * dh:D + (hh + 1) * dh]
            v = qkv[s, :, 2 * D + hh * dh:2 * D + (hh + 1) * dh]
            heads.append(masked_attention(q, k, v, masks[s][hh]))
        outs.append(torch.cat(heads, dim=1))
    o = torch.stack(outs)                                 # [S, L, D], heads side by side
    x1 = x0 + o @ w["w_o"].T
    h2 = layer_norm(x1, w["ln2_g"], w["ln2_b"])
    return x1 + gelu_tanh(h2 @ w["w_1"].T) @ w["w_2"].T


def block_forward_backward(bytes_, w: dict, masks, H: int, dy):
    """y and the gradients of <y, dy> for every weight (float64 numpy)."""
    wt = {k: torch.tensor(np.asarray(v, dtype=np.float64), requires_grad=True) for k, v in w.items()}
    y = block_forward(bytes_, wt, masks, H)
    (y * torch.as_tensor(np.asarray(dy, dtype=np.float64))).sum().backward()
    return y.detach().numpy(), {k: v.grad.numpy() for k, v in wt.items()}


def block_rows_forward(bytes_row, w: dict, block_masks, H: int, b: int, q_blocks):
    """y of one sample at the query blocks q_blocks only, float64 numpy.

    K and V need every token of the sample (LN1 and the K, V projections over
    the whole row); Q, the attention, the output projection and the MLP run
    for the requested blocks only, so full-length samples stay cheap.
    block_masks[h] is the bool [N, N] block mask of head h."""
    emb = np.asarray(w["emb"], dtype=np.float64)
    D = emb.shape[1]
    dh = D // H
    x0 = emb[np.asarray(bytes_row, dtype=np.int64)]
    t = torch.from_numpy

    def ln(x, g, bb):
        return layer_norm(t(x), t(np.asarray(g, np.float64)), t(np.asarray(bb, np.float64))).numpy()

    h = ln(x0, w["ln1_g"], w["ln1_b"])
    wqkv = np.asarray(w["w_qkv"], dtype=np.float64)
    k_all = h @ wqkv[D:2 * D].T
    v_all = h @ wqkv[2 * D:].T
    rows = np.concatenate([np.arange(i * b, (i + 1) * b) for i in q_blocks])
    q_all = np.zeros_like(k_all)
    q_all[rows] = h[rows] @ wqkv[:D].T
    o = np.zeros((len(x0), D))
    for hh in range(H):
        sl = slice(hh * dh, (hh + 1) * dh)
        oh, _ = oatt.forward(q_all[:, sl], k_all[:, sl], v_all[:, sl], block_masks[hh], b,
                             scale=1.0 / math.sqrt(dh), q_blocks=q_blocks)
        o[rows, sl] = oh[rows]
    x1 = x0[rows] + o[rows] @ np.asarray(w["w_o"], np.float64).T
    h2 = ln(x1, w["ln2_g"], w["ln2_b"])
    u = gelu_tanh(t(h2 @ np.asarray(w["w_1"], np.float64).T)).numpy()
    return rows, x1 + u @ np.asarray(w["w_2"], np.float64).T


def parameter_count(D: int, F: int) -> int:
    """Weights of one block plus the byte embedding."""
    return 256 * D + 4 * D + 3 * D * D + D * D + 2 * D * F
