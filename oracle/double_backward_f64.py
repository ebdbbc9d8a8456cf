"""Float64 CPU oracle of attention's backward-over-backward (test
infrastructure only, like attention_f64; the product path never uses it).

The FlashBoB listing ("Approaching I/O-optimality for Approximate
Attention", abstract) names the operation -- exact differentiation through
attention's backward pass -- and its structure: two row-wise scalars
determine every output through affine maps. The plain definition written
out here: the first backward is the map (Q, K, V, dO) -> (dQ, dK, dV) of
attention_f64 (dS = P o (dP - D), dQ = s dS K, dK = s dS^T Q, dV = P^T dO,
dP = dO V^T, D_i = sum_j P_ij dP_ij); given cotangents U_Q, U_K, U_V on its
outputs, backward-over-backward returns the gradient of

    L2 = <U_Q, dQ> + <U_K, dK> + <U_V, dV>

with respect to Q, K, V and dO. Writing M = s (U_Q K^T + Q U_K^T) (so that
the dQ and dK terms of L2 are <dS, M>) and differentiating term by term,
one head at a time, materialised:

    r_i   = sum_j P_ij M_ij                        (row scalar 1)
    E     = P o (M - r)                            (the part through dP)
    G     = M o (dP - D) - r dP + dO U_V^T         (dL2/dP, D's dependence included)
    g_i   = sum_j P_ij G_ij                        (row scalar 2)
    dS2   = P o (G - g)                            (through the softmax)

    gQ  = s (dS U_K + dS2 K)      gK = s (dS^T U_Q + dS2^T Q)
    gV  = E^T dO                  gdO = E V + P U_V

Masked scores have P = 0, so E, dS and dS2 vanish there. Pinned by
tests/test_oracle.py: central finite differences of L2 computed with
attention_f64.backward, and torch float64 double backward (autograd with
create_graph) of a separately written attention.
"""
from __future__ import annotations

import numpy as np

from .attention_f64 import forward_head, keep_mask


def double_backward_head(q, k, v, do, uq, uk, uv, scale, causal=True):
    """gQ, gK, gV, gdO of one head (all [N, d] float64), plus r and g."""
    q, k, v, do, uq, uk, uv = (np.asarray(a, np.float64) for a in (q, k, v, do, uq, uk, uv))
    n = q.shape[0]
    keep = keep_mask(n, n, causal)
    f = forward_head(q, k, v, scale, causal)
    P = f["P"]
    dP = do @ v.T
    D = (P * dP).sum(axis=1)
    dS = P * (dP - D[:, None])
    M = scale * (uq @ k.T + q @ uk.T)
    r = (P * M).sum(axis=1)
    E = P * (M - r[:, None])
    G = M * (dP - D[:, None]) - r[:, None] * dP + do @ uv.T
    G = np.where(keep, G, 0.0)
    g = (P * G).sum(axis=1)
    dS2 = P * (G - g[:, None])
    return {
        "gQ": scale * (dS @ uk + dS2 @ k),
        "gK": scale * (dS.T @ uq + dS2.T @ q),
        "gV": E.T @ do,
        "gdO": E @ v + P @ uv,
        "r": r, "g": g,
    }


def double_backward(q, k, v, do, uq, uk, uv, scale, causal=True):
    """Batched [B, H, N, d] form of double_backward_head."""
    q = np.asarray(q, np.float64)
    B, H = q.shape[:2]
    out = {name: np.empty(q.shape) for name in ("gQ", "gK", "gV", "gdO")}
    for b in range(B):
        for h in range(H):
            r = double_backward_head(q[b, h], k[b, h], v[b, h], do[b, h], uq[b, h], uk[b, h],
                                     uv[b, h], scale, causal)
            for name in out:
                out[name][b, h] = r[name]
    return out
