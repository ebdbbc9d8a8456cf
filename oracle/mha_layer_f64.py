"""Float64 CPU oracle of one causal multi-head attention layer (test
infrastructure only, like attention_f64; the product path never uses it).

The layer is the attention sublayer of the nanoGPT-shaped training step of
ddx issue #217 ("Backward of batched attention builds a contraction over every
pair of sequences and heads": one layer, 4 heads, 128 channels, 64 positions,
batch 12). The page names the model, not its algebra; the plainest reading,
taken here, is the usual one without biases, with x: [B, N, C], C = H * d:

    qkv = x W_qkv              [B, N, 3C]; channel block c of qkv is
                               q (c = 0), k (1), v (2), each [B, N, H, d]
    O   = attention(q, k, v)   causal, scale 1/sqrt(d)   -> [B, N, H, d]
    y   = O W_o                O read as [B, N, C]

and for a loss with dL/dy = dy:

    dO     = dy W_o^T,   dW_o   = sum over (b, n) of O^T dy
    dq, dk, dv = the attention backward (attention_f64.backward)
    dx     = dqkv W_qkv^T, dW_qkv = sum over (b, n) of x^T dqkv

The matrix products are numpy matmuls on float64; the attention is
attention_f64's. Pinned by tests/test_oracle.py against torch autograd in
float64 and by central finite differences on a tiny layer.
"""
from __future__ import annotations

import numpy as np

from .attention_f64 import backward as attention_backward
from .attention_f64 import forward as attention_forward


def _heads(t, H):
    """[B, N, C] -> [B, H, N, d]."""
    B, N, C = t.shape
    return t.reshape(B, N, H, C // H).transpose(0, 2, 1, 3)


def _merge(t):
    """[B, H, N, d] -> [B, N, C]."""
    B, H, N, d = t.shape
    return t.transpose(0, 2, 1, 3).reshape(B, N, H * d)


def layer(x, w_qkv, w_o, dy, H, causal=True):
    """Forward and backward of the layer. Returns y, dx, dW_qkv, dW_o and the
    intermediates qkv, O, LSE."""
    x, w_qkv, w_o, dy = (np.asarray(a, np.float64) for a in (x, w_qkv, w_o, dy))
    B, N, C = x.shape
    d = C // H
    qkv = x @ w_qkv
    q, k, v = (_heads(qkv[..., c * C:(c + 1) * C], H) for c in range(3))
    scale = 1.0 / np.sqrt(d)
    O, LSE = attention_forward(q, k, v, scale, causal)
    o_flat = _merge(O)
    y = o_flat @ w_o
    dO = _heads(dy @ w_o.T, H)
    g = attention_backward(q, k, v, dO, scale, causal)
    dqkv = np.concatenate([_merge(g[n]) for n in ("dQ", "dK", "dV")], axis=-1)
    dx = dqkv @ w_qkv.T
    dw_qkv = np.einsum("bnc,bne->ce", x, dqkv)
    dw_o = np.einsum("bnc,bne->ce", o_flat, dy)
    return {"y": y, "dx": dx, "dW_qkv": dw_qkv, "dW_o": dw_o, "qkv": qkv, "O": O, "LSE": LSE}
