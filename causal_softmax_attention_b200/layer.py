"""One causal multi-head attention layer, forward and backward, on one GPU.

The attention sublayer of the nanoGPT-shaped training step in ddx issue #217
("Backward of batched attention builds a contraction over every pair of
sequences and heads"), without biases, x: [B, N, C], C = H * d:

    qkv = x W_qkv            [B, N, 3C]: q, k, v are channel blocks 0, 1, 2,
                             each read in place as [B, N, H, d]
    O   = attention(q, k, v) causal, scale 1/sqrt(d), written as [B, N, C]
    y   = O W_o

    dO = dy W_o^T, dW_o = O^T dy (summed over batch and positions)
    dq, dk, dv -> one [B, N, 3C] array, dx = dqkv W_qkv^T, dW_qkv = x^T dqkv

The four projections are plain cuBLAS GEMMs (torch.matmul); the attention is
this library's attn_fwd_strided / attn_bwd_strided reading the projection
output and writing its gradient in place, so no head split or merge is ever
copied.
"""
from __future__ import annotations

import torch

from . import attn_bwd_strided, attn_bwd_workspace_bytes, attn_fwd_strided


def _qkv_views(t: torch.Tensor, H: int):
    B, N, C3 = t.shape
    d = C3 // (3 * H)
    t5 = t.view(B, N, 3, H, d)
    return tuple(t5[:, :, c].permute(0, 2, 1, 3) for c in range(3))


def _head_view(t: torch.Tensor, H: int):
    B, N, C = t.shape
    return t.view(B, N, H, C // H).permute(0, 2, 1, 3)


def layer_forward(x: torch.Tensor, w_qkv: torch.Tensor, w_o: torch.Tensor, H: int, stream=None):
    """y and the tensors the backward needs (x, qkv, O, LSE)."""
    B, N, C = x.shape
    if C % H or w_qkv.shape != (C, 3 * C) or w_o.shape != (C, C):
        raise ValueError("expected x [B, N, C], w_qkv [C, 3C], w_o [C, C], C divisible by H")
    d = C // H
    qkv = x @ w_qkv
    q, k, v = _qkv_views(qkv, H)
    o = torch.empty(B, N, C, dtype=x.dtype, device=x.device)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=x.device)
    attn_fwd_strided(q, k, v, _head_view(o, H), lse, True, d ** -0.5, stream)
    return o @ w_o, (x, qkv, o, lse)


def layer_backward(dy: torch.Tensor, saved, w_qkv: torch.Tensor, w_o: torch.Tensor, H: int,
                   workspace: torch.Tensor | None = None, stream=None):
    """dx, dW_qkv, dW_o for dL/dy = dy."""
    x, qkv, o, lse = saved
    B, N, C = x.shape
    d = C // H
    do = dy @ w_o.T
    dqkv = torch.empty_like(qkv)
    q, k, v = _qkv_views(qkv, H)
    dq, dk, dv = _qkv_views(dqkv, H)
    if workspace is None:
        workspace = torch.empty(attn_bwd_workspace_bytes(B, H, N, d, x.dtype), dtype=torch.uint8,
                                device=x.device)
    attn_bwd_strided(q, k, v, _head_view(o, H), _head_view(do, H), lse, dq, dk, dv, workspace,
                     True, d ** -0.5, stream)
    dx = dqkv @ w_qkv.T
    dw_qkv = x.reshape(-1, C).T @ dqkv.reshape(-1, 3 * C)
    dw_o = o.reshape(-1, C).T @ dy.reshape(-1, C)
    return dx, dw_qkv, dw_o
