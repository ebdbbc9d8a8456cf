"""Float64 CPU oracle for batched, multi-head, causal softmax attention.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or links
this module: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference arm use it. It shares no code with the CUDA library.

What it computes is the plain materialised definition, one (b, h) head at a
time, in numpy float64:

* scores ``S = scale * Q K^T`` with the causal filter ``i >= j`` (diagonal
  kept) -- ddx issue #217, repro, the ``scores`` CTE (``WHERE q.pos >= k.pos``,
  ``SUM(q.val * k.val) / 2.0``) and its JAX restatement (``tril`` mask);
* the max-shifted softmax ``w = exp(S - max_j S)``, ``z = sum_j w``,
  ``P = w / z`` -- same repro, the ``weights`` and ``norm`` CTEs;
* ``O = P V`` -- same repro, the ``heads`` CTE;
* one saved number per row, ``LSE = m + log z`` -- ddx issue #243, item 2;
* the backward with the shift's gradient dropped (ddx issue #243, item 1:
  the MAX terms sum to zero because the shift cancels in w / z):
  ``dV = P^T dO``, ``dP = dO V^T``, ``D_i = sum_c dO_ic O_ic`` (the "sums
  weighted by the softmax" of issue #243 item 2), ``dS = P o (dP - D)``,
  ``dQ = scale dS K``, ``dK = scale dS^T Q`` -- ddx PR #162, "What changed"
  (transpose p = w / z per score, then p @ v);
* the backward *with* the shift, differentiating through w, z and m
  explicitly, used only to check that the shift's gradient cancels.

Masked scores are excluded with a boolean mask (P is exactly 0 there), never
with an additive large negative number. Besides the causal and full filters,
any boolean mask can be given, and ``block_mask_keep`` expands a block mask
(one kind per 128 x 128 tile: none, all, or causal inside the tile) into one.

Pins (tests/test_oracle.py): central finite differences, softmax
normalisation, invariance to a per-row score shift, with-shift == without-shift
backward, closed forms (N = 1, Q = 0, equal V rows), row/column identities, a
float64 torch-autograd cross-check of a separately written formula, and the
causal pair count printed by the ddx issue #217 repro. Every function here is
pinned by at least one of them.
"""
from __future__ import annotations

import numpy as np


def keep_mask(n_q: int, n_k: int, causal: bool, q_offset: int = 0) -> np.ndarray:
    """Boolean [n_q, n_k] mask of the scores that take part (True = kept).

    Query row r stands for position ``q_offset + r``; key column j for
    position j. The causal filter keeps ``pos_q >= pos_k`` (ddx issue #217,
    repro: ``WHERE q.pos >= k.pos``), so each row keeps its diagonal.
    """
    if not causal:
        return np.ones((n_q, n_k), dtype=bool)
    i = q_offset + np.arange(n_q)[:, None]
    j = np.arange(n_k)[None, :]
    return i >= j


def block_mask_keep(block_mask, n: int, tile: int = 128) -> np.ndarray:
    """Boolean [n, n] mask of the scores kept under a block mask.

    ``block_mask[a, b]`` describes the tile of query rows [a*tile, (a+1)*tile)
    and key columns [b*tile, (b+1)*tile): 0 keeps none of its scores, 1 keeps
    all of them, 2 keeps those whose key lies at or before the query inside
    the tile (local key index <= local query index). The causal filter is the
    instance 1 below the diagonal, 2 on it, 0 above: the block-sparse
    generalisation of the mask that ddx PR #162 applies as a filter on the
    grouping keys.
    """
    bm = np.asarray(block_mask)
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    kind = bm[i // tile, j // tile]
    return (kind == 1) | ((kind == 2) & (j % tile <= i % tile))


def forward_head(q, k, v, scale, causal=True, row_shift=None, keep=None, q_offset=0):
    """Forward of one head. q: [N_q, d], k, v: [N_k, d] float64.

    Returns a dict with S (scores, including ``row_shift`` if given), keep,
    m (row max over kept scores), w, z, P, O and LSE = m + log z.

    ``row_shift`` (length-N, optional) is added to row i of the scores before
    the softmax; it exists only to test the invariance of everything but LSE
    to such a shift. ``keep`` (boolean [N_q, N_k], optional) replaces the
    causal / full filter; a row that keeps no score has P = 0, O = 0 and
    LSE = -inf (the log of an empty sum). With N_q != N_k the causal filter
    reads query row r as position ``q_offset + r`` and key column j as
    position j (the repro's ``WHERE q.pos >= k.pos`` on absolute positions).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    n = q.shape[0]
    S = scale * (q @ k.T)
    if row_shift is not None:
        S = S + np.asarray(row_shift, np.float64)[:, None]
    keep = keep_mask(n, k.shape[0], causal, q_offset) if keep is None else np.asarray(keep, bool)
    m = np.where(keep, S, -np.inf).max(axis=1)
    w = np.zeros_like(S)
    w[keep] = np.exp((S - m[:, None])[keep])
    z = w.sum(axis=1)
    empty = z == 0
    P = w / np.where(empty, 1.0, z)[:, None]
    O = P @ v
    with np.errstate(divide="ignore"):
        LSE = np.where(empty, -np.inf, m + np.log(np.where(empty, 1.0, z)))
    return {"S": S, "keep": keep, "m": m, "w": w, "z": z, "P": P, "O": O, "LSE": LSE}


def backward_head(q, k, v, do, scale, causal=True, row_shift=None, keep=None, q_offset=0):
    """Backward of one head without the shift's gradient (q, do: [N_q, d];
    k, v: [N_k, d]; the filter as in forward_head).

    Returns dict(dQ, dK, dV, D, D_rows, dS, fwd) where D = sum_c dO o O (the
    form the GPU uses) and D_rows = sum_j P o dP (the softmax-weighted sum of
    ddx issue #243 item 2); the two agree up to rounding.
    """
    f = forward_head(q, k, v, scale, causal, row_shift, keep, q_offset)
    do = np.asarray(do, np.float64)
    k = np.asarray(k, np.float64)
    q = np.asarray(q, np.float64)
    v = np.asarray(v, np.float64)
    P, O = f["P"], f["O"]
    dV = P.T @ do
    dP = do @ v.T
    D = (do * O).sum(axis=1)
    D_rows = (P * dP).sum(axis=1)
    dS = P * (dP - D[:, None])
    dQ = scale * (dS @ k)
    dK = scale * (dS.T @ q)
    return {"dQ": dQ, "dK": dK, "dV": dV, "D": D, "D_rows": D_rows, "dS": dS, "fwd": f}


def backward_head_with_shift(q, k, v, do, scale, causal=True, row_shift=None,
                             ties="first"):
    """Backward of one head that keeps the max-shift's gradient.

    Differentiates the window spelling of ddx issue #217's repro term by term:
    P = w / z, z = sum_j w, w = exp(S - m), m = max_j S. The gradient of m
    is routed to the argmax column of each row (``ties='first'``: first
    maximal column; ``ties='split'``: shared evenly among tied columns).
    Mathematically the routed terms sum to zero (ddx issue #243, item 1).
    """
    f = forward_head(q, k, v, scale, causal, row_shift)
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    w, z, S, keep = f["w"], f["z"], f["S"], f["keep"]
    dV = f["P"].T @ do
    dP = do @ v.T
    # P_ik = w_ik / z_i  =>  dL/dw_ij = dP_ij / z_i - sum_k dP_ik w_ik / z_i^2
    dw = dP / z[:, None] - ((dP * w).sum(axis=1) / z**2)[:, None]
    dw = np.where(keep, dw, 0.0)
    # w_ij = exp(S_ij - m_i)
    dS = dw * w
    dm = -(dw * w).sum(axis=1)
    # m_i = max_j S_ij over kept j
    Sk = np.where(keep, S, -np.inf)
    if ties == "first":
        am = Sk.argmax(axis=1)
        dS[np.arange(S.shape[0]), am] += dm
    else:
        tied = Sk == Sk.max(axis=1)[:, None]
        dS += tied * (dm / tied.sum(axis=1))[:, None]
    dQ = scale * (dS @ k)
    dK = scale * (dS.T @ q)
    return {"dQ": dQ, "dK": dK, "dV": dV, "dm": dm, "dS": dS}


def forward(q, k, v, scale, causal=True, keep=None, q_offset=0):
    """Batched forward. q: [B, H, N_q, d], k, v: [B, H, N_k, d]. Returns
    O [B,H,N_q,d], LSE [B,H,N_q]. ``keep`` (boolean [N_q, N_k], optional) is
    shared by every head; ``q_offset`` as in forward_head."""
    q = np.asarray(q, np.float64)
    B, H, N, d = q.shape
    O = np.empty((B, H, N, v.shape[-1]))
    LSE = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            f = forward_head(q[b, h], k[b, h], v[b, h], scale, causal, keep=keep,
                             q_offset=q_offset)
            O[b, h] = f["O"]
            LSE[b, h] = f["LSE"]
    return O, LSE


def backward(q, k, v, do, scale, causal=True, keep=None, q_offset=0):
    """Batched backward. Returns dQ, O [B,H,N_q,d], dK, dV [B,H,N_k,d], LSE
    and D [B,H,N_q]. ``keep`` (boolean [N_q, N_k], optional) is shared by
    every head; ``q_offset`` as in forward_head."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    B, H, N, d = q.shape
    out = {name: np.empty(q.shape) for name in ("dQ", "O")}
    out.update({name: np.empty(k.shape) for name in ("dK", "dV")})
    out["LSE"] = np.empty((B, H, N))
    out["D"] = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            r = backward_head(q[b, h], k[b, h], v[b, h], do[b, h], scale, causal, keep=keep,
                              q_offset=q_offset)
            for name in ("dQ", "dK", "dV", "D"):
                out[name][b, h] = r[name]
            out["O"][b, h] = r["fwd"]["O"]
            out["LSE"][b, h] = r["fwd"]["LSE"]
    return out


def query_rows(q, k, v, do, scale, rows, causal=True):
    """O, LSE, D and dQ of selected query rows of one head, each from its definition.

    Row i of the scores only needs q_i and the keys it keeps, so these rows
    are exact without the rest of the N x N table. q, k, v, do: [N, d].
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    rows = np.asarray(rows)
    n, d = q.shape
    res = {"O": np.empty((len(rows), v.shape[1])), "LSE": np.empty(len(rows)),
           "D": np.empty(len(rows)), "dQ": np.empty((len(rows), d))}
    for r, i in enumerate(rows):
        last = i + 1 if causal else n
        s = scale * (k[:last] @ q[i])
        m = s.max()
        w = np.exp(s - m)
        z = w.sum()
        p = w / z
        o = p @ v[:last]
        dp = v[:last] @ do[i]
        Di = do[i] @ o
        ds = p * (dp - Di)
        res["O"][r] = o
        res["LSE"][r] = m + np.log(z)
        res["D"][r] = Di
        res["dQ"][r] = scale * (ds @ k[:last])
    return res


def backward_row_block(q, k, v, do, scale, r0, r1, causal=True):
    """The backward's terms contributed by query rows [r0, r1) of one head.

    dK and dV are sums over query rows, so the full backward is the sum of
    these blocks over a partition of the rows; dQ, O, LSE and D of the
    block's rows are complete. Returns dQ [r1-r0, d] and the block's
    contributions dK, dV [N, d] (zero for keys the block never sees), plus
    O, LSE, D of the rows. Used where the N x N table does not fit in memory.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    n = q.shape[0]
    last = r1 if causal else n          # keys this block can see
    S = scale * (q[r0:r1] @ k[:last].T)
    keep = keep_mask(r1 - r0, last, causal, q_offset=r0)
    m = np.where(keep, S, -np.inf).max(axis=1)
    w = np.zeros_like(S)
    w[keep] = np.exp((S - m[:, None])[keep])
    z = w.sum(axis=1)
    P = w / z[:, None]
    O = P @ v[:last]
    dob = do[r0:r1]
    dP = dob @ v[:last].T
    D = (dob * O).sum(axis=1)
    dS = P * (dP - D[:, None])
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    dK[:last] = scale * (dS.T @ q[r0:r1])
    dV[:last] = P.T @ dob
    return {"dQ": scale * (dS @ k[:last]), "dK": dK, "dV": dV,
            "O": O, "LSE": m + np.log(z), "D": D}


def backward_blocked(q, k, v, do, scale, causal=True, rows_per_block=1024):
    """The whole backward of one head as the sum of its row blocks.

    Runs ``backward_row_block`` over consecutive blocks of query rows and adds
    up their dK, dV contributions (dK and dV are sums over query rows); dQ, O,
    LSE and D of each block's rows are complete as they come. The result is
    ``backward_head``'s without ever holding more than rows_per_block x N of
    the score table. q, k, v, do: [N, d] float64.
    """
    n, d = np.asarray(q).shape
    out = {"dQ": np.empty((n, d)), "dK": np.zeros((n, d)), "dV": np.zeros((n, d)),
           "O": np.empty((n, np.asarray(v).shape[1])), "LSE": np.empty(n), "D": np.empty(n)}
    for r0 in range(0, n, rows_per_block):
        r1 = min(n, r0 + rows_per_block)
        blk = backward_row_block(q, k, v, do, scale, r0, r1, causal)
        out["dK"] += blk["dK"]
        out["dV"] += blk["dV"]
        for name in ("dQ", "O", "LSE", "D"):
            out[name][r0:r1] = blk[name]
    return out


def key_tail(q, k, v, do, scale, j0, rows_per_block=None):
    """dK and dV of keys j >= j0 of one causal head.

    Under the causal filter key j only meets query rows i >= j, so the tail
    needs rows j0..N-1 only (each row's softmax is still over all its keys).
    rows_per_block splits those rows into blocks whose dK, dV contributions
    are summed (the same sums over the same rows, holding rows_per_block x N
    of the score table at a time instead of (N - j0) x N).
    """
    n = q.shape[0]
    step = (n - j0) if rows_per_block is None else rows_per_block
    dk = np.zeros((n - j0, np.asarray(k).shape[1]))
    dv = np.zeros((n - j0, np.asarray(v).shape[1]))
    for r0 in range(j0, n, step):
        blk = backward_row_block(q, k, v, do, scale, r0, min(r0 + step, n), causal=True)
        dk += blk["dK"][j0:]
        dv += blk["dV"][j0:]
    return {"dK": dk, "dV": dv}


def causal_pair_count(B: int, H: int, N: int) -> int:
    """Number of (b, h, i, j) scores the causal filter keeps, counted from the mask."""
    return B * H * int(keep_mask(N, N, True).sum())
