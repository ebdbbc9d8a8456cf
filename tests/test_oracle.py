"""Pins of the float64 oracle against what the pages and the mathematics fix.

None of these compare the oracle with itself: finite differences, closed
forms, invariants, the pair count printed by ddx issue #217's repro and an
independently written torch float64 autograd formula. The last group plants
plausible mistakes in copies of the oracle's backward and checks that the
finite-difference pin catches each of them.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention_f64 as A
from seeded_inputs import ddx_issue217_input

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def rel(a, b):
    """Normwise relative error max|a-b| / max|b|."""
    a, b = np.asarray(a), np.asarray(b)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def loss_fn(q, k, v, do, scale, causal):
    return float((do * A.forward_head(q, k, v, scale, causal)["O"]).sum())


def fd_grads(q, k, v, do, scale, causal, h=1e-6):
    """Central finite differences of L = sum(dO o O(q, k, v))."""
    out = []
    for which in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(args[which])
        for idx in np.ndindex(g.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            g[idx] = (loss_fn(*plus, do, scale, causal) - loss_fn(*minus, do, scale, causal)) / (2 * h)
        out.append(g)
    return out


def tiny_case(seed=0, n=8, d=4):
    return rnd(seed, n, d), rnd(seed + 1, n, d), rnd(seed + 2, n, d), rnd(seed + 3, n, d)


# --------------------------------------------------------------------------
# finite differences (B=1, H=1, N=8, d=4)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [True, False])
def test_finite_differences(causal):
    q, k, v, do = tiny_case()
    scale = 0.5
    r = A.backward_head(q, k, v, do, scale, causal)
    fq, fk, fv = fd_grads(q, k, v, do, scale, causal)
    for an, fd in ((r["dQ"], fq), (r["dK"], fk), (r["dV"], fv)):
        assert np.all(np.abs(an - fd) <= 1e-7 * np.abs(fd).max() + 1e-9)


# --------------------------------------------------------------------------
# softmax normalisation and the causal filter
# --------------------------------------------------------------------------
def test_softmax_rows_sum_to_one_and_mask_is_exact():
    q, k, v, _ = tiny_case(5, n=33, d=16)
    f = A.forward_head(q, k, v, 0.25, causal=True)
    P = f["P"]
    assert np.abs(P.sum(axis=1) - 1).max() <= 1e-14
    iu = np.triu_indices(33, 1)
    assert np.all(P[iu] == 0.0)
    il = np.tril_indices(33)
    assert np.all(P[il] > 0.0)


def test_lse_is_log_of_normaliser():
    q, k, v, _ = tiny_case(6, n=20, d=8)
    f = A.forward_head(q, k, v, 0.3, causal=True)
    S = 0.3 * q @ k.T
    for i in range(20):
        assert abs(f["LSE"][i] - np.log(np.exp(S[i, : i + 1]).sum())) < 1e-13


# --------------------------------------------------------------------------
# invariance to a per-row shift of the scores
# --------------------------------------------------------------------------
def test_row_shift_invariance():
    q, k, v, do = tiny_case(7, n=24, d=8)
    c = rnd(11, 24) * 10
    c[0], c[1] = 50.0, -50.0
    a = A.backward_head(q, k, v, do, 0.4, True)
    b = A.backward_head(q, k, v, do, 0.4, True, row_shift=c)
    assert rel(b["fwd"]["O"], a["fwd"]["O"]) <= 1e-12
    assert np.abs(b["fwd"]["LSE"] - c - a["fwd"]["LSE"]).max() <= 1e-12 * 50
    for g in ("dQ", "dK", "dV"):
        assert rel(b[g], a[g]) <= 1e-12


# --------------------------------------------------------------------------
# the shift's gradient cancels (ddx issue #243, item 1)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("ties", ["first", "split"])
@pytest.mark.parametrize("causal", [True, False])
def test_with_shift_equals_without(ties, causal):
    q, k, v, do = tiny_case(8, n=40, d=16)
    a = A.backward_head(q, k, v, do, 0.25, causal)
    b = A.backward_head_with_shift(q, k, v, do, 0.25, causal, ties=ties)
    for g in ("dQ", "dK", "dV"):
        assert rel(b[g], a[g]) <= 1e-12
    # the routed max-terms are tiny rounding residue, not signal
    assert np.abs(b["dm"]).max() <= 1e-13


def test_with_shift_ties_split_equals_first():
    # identical keys make every row's maximum tied
    q, _, v, do = tiny_case(9, n=12, d=4)
    k = np.tile(rnd(10, 1, 4), (12, 1))
    a = A.backward_head_with_shift(q, k, v, do, 0.5, True, ties="first")
    b = A.backward_head_with_shift(q, k, v, do, 0.5, True, ties="split")
    for g in ("dQ", "dK", "dV"):
        assert np.abs(a[g] - b[g]).max() <= 1e-12 * max(1.0, np.abs(a[g]).max())


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------
def test_single_position():
    q, k, v, do = tiny_case(12, n=1, d=8)
    r = A.backward_head(q, k, v, do, 0.3, True)
    assert np.array_equal(r["fwd"]["O"], v)
    assert np.allclose(r["dV"], do, rtol=0, atol=1e-15)
    assert np.abs(r["dQ"]).max() <= 1e-14 and np.abs(r["dK"]).max() <= 1e-14


def test_zero_queries_give_prefix_means():
    n, d = 17, 5
    _, k, v, do = tiny_case(13, n=n, d=d)
    q = np.zeros((n, d))
    r = A.backward_head(q, k, v, do, 0.7, True)
    f = r["fwd"]
    for i in range(n):
        assert np.allclose(f["P"][i, : i + 1], 1.0 / (i + 1), rtol=1e-14, atol=0)
        assert np.allclose(f["O"][i], v[: i + 1].mean(axis=0), rtol=1e-13, atol=1e-15)
        assert abs(f["LSE"][i] - np.log(i + 1)) <= 1e-14
    want_dv = np.array([sum(do[i] / (i + 1) for i in range(j, n)) for j in range(n)])
    assert np.allclose(r["dV"], want_dv, rtol=1e-13, atol=1e-15)


def test_equal_value_rows_give_zero_score_gradients():
    n, d = 21, 6
    q, k, _, do = tiny_case(14, n=n, d=d)
    v = np.tile(rnd(15, 1, d), (n, 1))
    r = A.backward_head(q, k, v, do, 0.5, True)
    assert np.allclose(r["fwd"]["O"], v, rtol=1e-14, atol=1e-14)
    assert np.abs(r["dQ"]).max() <= 1e-13
    assert np.abs(r["dK"]).max() <= 1e-13


# --------------------------------------------------------------------------
# row and column identities
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [True, False])
def test_identities(causal):
    q, k, v, do = tiny_case(16, n=50, d=12)
    r = A.backward_head(q, k, v, do, 0.3, causal)
    scale_g = np.abs(r["dK"]).max()
    assert np.abs(r["dK"].sum(axis=0)).max() <= 1e-12 * 50 * scale_g
    assert np.allclose(r["dV"].sum(axis=0), do.sum(axis=0), rtol=1e-12, atol=1e-12)
    assert np.allclose(r["D"], r["D_rows"], rtol=1e-12, atol=1e-13)
    assert np.abs(r["dS"].sum(axis=1)).max() <= 1e-13


# --------------------------------------------------------------------------
# independent float64 cross-check: torch autograd of a separately written formula
# --------------------------------------------------------------------------
def torch_reference(q, k, v, do, scale, causal):
    q, k, v = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    s = (q @ k.transpose(-1, -2)) * scale
    if causal:
        n = q.shape[-2]
        s = s.masked_fill(~torch.ones(n, n, dtype=torch.bool).tril(), float("-inf"))
    o = torch.softmax(s, dim=-1) @ v
    (o * torch.tensor(do)).sum().backward()
    return o.detach().numpy(), q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("causal", [True, False])
def test_torch_autograd_cross_check(causal):
    B, H, N, d = 2, 3, 37, 16
    q, k, v, do = (rnd(20 + t, B, H, N, d) for t in range(4))
    out = A.backward(q, k, v, do, 0.25, causal)
    o, gq, gk, gv = torch_reference(q, k, v, do, 0.25, causal)
    assert rel(out["O"], o) <= 1e-12
    assert rel(out["dQ"], gq) <= 1e-12
    assert rel(out["dK"], gk) <= 1e-12
    assert rel(out["dV"], gv) <= 1e-12


# --------------------------------------------------------------------------
# N_q != N_k: query row r at position q_offset + r, key j at position j
# --------------------------------------------------------------------------
def torch_reference_positions(q, k, v, do, scale, causal, q_offset):
    """Separately written: scores masked by explicit positions (row r is
    position q_offset + r), softmax, weighted values; torch float64 autograd."""
    q, k, v = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    s = (q @ k.transpose(-1, -2)) * scale
    if causal:
        pos_q = q_offset + torch.arange(q.shape[-2])
        pos_k = torch.arange(k.shape[-2])
        s = s.masked_fill(pos_q[:, None] < pos_k[None, :], float("-inf"))
    o = torch.softmax(s, dim=-1) @ v
    (o * torch.tensor(do)).sum().backward()
    return o.detach().numpy(), q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("nq,nk,off,causal", [(5, 8, 3, True), (8, 5, 0, True), (6, 9, 0, False),
                                              (4, 7, 1, True)])
def test_rectangular_finite_differences(nq, nk, off, causal):
    rng = np.random.default_rng(nq * 100 + nk)
    q, do = rng.standard_normal((nq, 4)), rng.standard_normal((nq, 4))
    k, v = rng.standard_normal((nk, 4)), rng.standard_normal((nk, 4))
    r = A.backward_head(q, k, v, do, 0.5, causal, q_offset=off)
    h = 1e-6

    def loss(q_, k_, v_):
        return float((do * A.forward_head(q_, k_, v_, 0.5, causal, q_offset=off)["O"]).sum())

    for which, name in ((0, "dQ"), (1, "dK"), (2, "dV")):
        args = [q, k, v]
        g = np.zeros_like(args[which])
        for idx in np.ndindex(g.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        assert np.abs(g - r[name]).max() <= 1e-7 * max(1.0, np.abs(r[name]).max()), name


@pytest.mark.parametrize("nq,nk,off,causal", [(37, 70, 33, True), (70, 37, 0, True),
                                              (20, 50, 5, True), (33, 21, 0, False)])
def test_rectangular_torch_autograd_cross_check(nq, nk, off, causal):
    q, do = rnd(40, 2, 3, nq, 16), rnd(41, 2, 3, nq, 16)
    k, v = rnd(42, 2, 3, nk, 16), rnd(43, 2, 3, nk, 16)
    out = A.backward(q, k, v, do, 0.25, causal, q_offset=off)
    o, gq, gk, gv = torch_reference_positions(q, k, v, do, 0.25, causal, off)
    assert out["dK"].shape == k.shape and out["dQ"].shape == q.shape
    assert rel(out["O"], o) <= 1e-12
    assert rel(out["dQ"], gq) <= 1e-12
    assert rel(out["dK"], gk) <= 1e-12
    assert rel(out["dV"], gv) <= 1e-12


def test_rectangular_is_a_row_block_of_the_square_problem():
    # the last n_q rows of a square causal head, offset n - n_q: the same O,
    # LSE, dQ rows, and dK, dV equal to those rows' contributions
    # (backward_row_block, pinned above against the materialised head)
    n, nq, d = 90, 23, 8
    q, k, v, do = tiny_case(50, n=n, d=d)
    r = A.backward_head(q[n - nq:], k, v, do[n - nq:], 0.4, True, q_offset=n - nq)
    blk = A.backward_row_block(q, k, v, do, 0.4, n - nq, n, True)
    for name in ("dQ", "dK", "dV", "D"):
        assert rel(r[name], blk[name]) <= 1e-12, name
    assert rel(r["fwd"]["O"], blk["O"]) <= 1e-12
    assert np.allclose(r["fwd"]["LSE"], blk["LSE"], rtol=1e-13)


def test_rectangular_special_cases():
    q, k, v, do = tiny_case(60, n=12, d=4)
    # square with offset 0 is the square causal problem
    a = A.backward_head(q, k, v, do, 0.3, True, q_offset=0)
    b = A.backward_head(q, k, v, do, 0.3, True)
    assert all(np.array_equal(a[n], b[n]) for n in ("dQ", "dK", "dV"))
    # an offset past the last key makes the causal filter keep everything
    c = A.backward_head(q[:5], k, v, do[:5], 0.3, True, q_offset=11)
    e = A.backward_head(q[:5], k, v, do[:5], 0.3, False)
    assert all(np.array_equal(c[n], e[n]) for n in ("dQ", "dK", "dV"))
    # keys no query can see get zero gradients
    f = A.backward_head(q[:3], k, v, do[:3], 0.3, True, q_offset=4)
    assert np.count_nonzero(f["dK"][7:]) == 0 and np.count_nonzero(f["dV"][7:]) == 0


# --------------------------------------------------------------------------
# ddx issue #217's repro: its printed table sizes and its float64 JAX check
# --------------------------------------------------------------------------
def test_ddx_issue217_repro():
    with open(os.path.join(GOLDEN, "ddx_issue217_repro.json")) as fh:
        g = json.load(fh)
    inp, printed = g["input"], g["printed"]
    S, T, H, C = inp["S_sequences"], inp["T_positions"], inp["H_heads"], inp["C_channels"]
    q, k, v = ddx_issue217_input(S, T, H, C)
    assert q.shape == (S, H, T, C)
    # the scores table keeps S*H*T(T+1)/2 rows
    assert oracle.causal_pair_count(S, H, T) == printed["causal_score_rows"]
    assert (S * H * T) ** 2 == printed["cross_product_rows"]
    assert S * H * T * T == printed["seq_head_pos_pos"]
    scale = 1.0 / inp["score_divisor"]
    O, _ = A.forward(q, k, v, scale, True)
    assert O.size == printed["saved_2_rows_attention_output"]
    # loss sum(O^2)/2 => dO = O; check the gradient at the repro's tolerances
    out = A.backward(q, k, v, O, scale, True)
    _, gq, gk, gv = torch_reference(q, k, v, O, scale, True)
    tol = printed["jax_check"]
    for ours, ref in ((out["dQ"], gq), (out["dK"], gk), (out["dV"], gv)):
        assert np.allclose(ours, ref, rtol=tol["rtol"], atol=tol["atol"])


# --------------------------------------------------------------------------
# row-wise, row-block and key-tail forms against the materialised head
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [True, False])
def test_query_rows_and_row_blocks(causal):
    n, d = 70, 8
    q, k, v, do = tiny_case(30, n=n, d=d)
    full = A.backward_head(q, k, v, do, 0.35, causal)
    rows = [0, 1, 17, 63, 69]
    qr = A.query_rows(q, k, v, do, 0.35, rows, causal)
    assert rel(qr["dQ"], full["dQ"][rows]) <= 1e-12
    assert rel(qr["O"], full["fwd"]["O"][rows]) <= 1e-12
    assert np.allclose(qr["LSE"], full["fwd"]["LSE"][rows], rtol=1e-13)
    assert np.allclose(qr["D"], full["D"][rows], rtol=1e-12, atol=1e-13)
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    for r0 in range(0, n, 16):
        blk = A.backward_row_block(q, k, v, do, 0.35, r0, min(n, r0 + 16), causal)
        dK += blk["dK"]
        dV += blk["dV"]
        assert rel(blk["dQ"], full["dQ"][r0:r0 + 16]) <= 1e-12
    assert rel(dK, full["dK"]) <= 1e-12
    assert rel(dV, full["dV"]) <= 1e-12
    if causal:
        tail = A.key_tail(q, k, v, do, 0.35, 50)
        assert rel(tail["dK"], full["dK"][50:]) <= 1e-12
        assert rel(tail["dV"], full["dV"][50:]) <= 1e-12
        # the same tail from row blocks (a ragged last block included)
        tail = A.key_tail(q, k, v, do, 0.35, 50, rows_per_block=7)
        assert rel(tail["dK"], full["dK"][50:]) <= 1e-12
        assert rel(tail["dV"], full["dV"][50:]) <= 1e-12


@pytest.mark.parametrize("causal,block", [(True, 16), (True, 23), (False, 16), (True, 1000)])
def test_blocked_backward_equals_the_materialised_head(causal, block):
    # the sum of the row blocks, whatever the block size (ragged last block,
    # one block for everything), is the materialised head's backward
    n, d = 70, 8
    q, k, v, do = tiny_case(31, n=n, d=d)
    full = A.backward_head(q, k, v, do, 0.35, causal)
    got = A.backward_blocked(q, k, v, do, 0.35, causal, rows_per_block=block)
    for name in ("dQ", "dK", "dV", "D"):
        assert rel(got[name], full[name]) <= 1e-12, name
    assert rel(got["O"], full["fwd"]["O"]) <= 1e-12
    assert np.allclose(got["LSE"], full["fwd"]["LSE"], rtol=1e-13)


def test_batched_equals_per_head_and_head_permutation():
    B, H, N, d = 2, 3, 19, 4
    q, k, v, do = (rnd(40 + t, B, H, N, d) for t in range(4))
    out = A.backward(q, k, v, do, 0.5, True)
    perm = [2, 0, 1]
    outp = A.backward(q[:, perm], k[:, perm], v[:, perm], do[:, perm], 0.5, True)
    for g in ("dQ", "dK", "dV", "O", "LSE"):
        assert np.array_equal(outp[g], out[g][:, perm])


# --------------------------------------------------------------------------
# test of the tests: plausible mistakes planted in copies of the backward
# --------------------------------------------------------------------------
def _mutant(kind):
    def bwd(q, k, v, do, scale, causal):
        f = A.forward_head(q, k, v, scale, causal)
        P, O = f["P"], f["O"]
        dV = P.T @ do
        dP = do @ v.T
        D = (do * O).sum(axis=1)
        if kind == "drop_D":
            dS = P * dP
        elif kind == "sign":
            dS = P * (dP + D[:, None])
        else:
            dS = P * (dP - D[:, None])
        dQ = scale * dS @ k
        dK = scale * dS.T @ q
        if kind == "transpose_dV":
            dV = P @ do
        if kind == "no_scale_dK":
            dK = dS.T @ q
        if kind == "swap_dQ_operand":
            dQ = scale * dS.T @ k
        return {"dQ": dQ, "dK": dK, "dV": dV}
    return bwd


@pytest.mark.parametrize("kind", ["drop_D", "sign", "transpose_dV", "no_scale_dK", "swap_dQ_operand"])
def test_finite_differences_catch_planted_mistakes(kind):
    q, k, v, do = tiny_case()
    r = _mutant(kind)(q, k, v, do, 0.5, True)
    fq, fk, fv = fd_grads(q, k, v, do, 0.5, True)
    worst = max(rel(r["dQ"], fq), rel(r["dK"], fk), rel(r["dV"], fv))
    assert worst > 1e-3


def test_pair_count_catches_a_mask_without_diagonal(monkeypatch):
    def strict(n_q, n_k, causal, q_offset=0):
        i = q_offset + np.arange(n_q)[:, None]
        return (i > np.arange(n_k)[None, :]) if causal else np.ones((n_q, n_k), bool)
    monkeypatch.setattr(A, "keep_mask", strict)
    assert A.causal_pair_count(3, 2, 8) != 216


# --------------------------------------------------------------------------
# general and block masks (block-sparse attention)
# --------------------------------------------------------------------------
def causal_block_mask(n, tile=128):
    t = -(-n // tile)
    a = np.arange(t)
    return np.where(a[:, None] > a[None, :], 1, np.where(a[:, None] == a[None, :], 2, 0))


@pytest.mark.parametrize("n", [1, 5, 128, 130, 257, 640])
def test_block_mask_expands_causal_and_full(n):
    assert np.array_equal(A.block_mask_keep(causal_block_mask(n), n), A.keep_mask(n, n, True))
    t = -(-n // 128)
    assert A.block_mask_keep(np.ones((t, t), int), n).all()
    assert not A.block_mask_keep(np.zeros((t, t), int), n).any()


def test_block_mask_kind_two_off_the_diagonal():
    # kind 2 keeps local key <= local query inside any tile, not only on the diagonal
    bm = np.array([[0, 0], [2, 0]])
    keep = A.block_mask_keep(bm, 200)
    assert keep[128 + 5, 5] and keep[128 + 5, 0] and not keep[128 + 5, 6]
    assert not keep[:128].any() and not keep[:, 128:].any()


def masked_loss(q, k, v, do, scale, keep):
    return float((do * A.forward_head(q, k, v, scale, keep=keep)["O"]).sum())


def test_finite_differences_under_a_mask_with_an_empty_row():
    q, k, v, do = tiny_case(seed=40)
    rng = np.random.default_rng(41)
    keep = rng.random((8, 8)) < 0.5
    keep[np.arange(8), rng.integers(0, 8, 8)] = True
    keep[3] = False  # a row that keeps nothing
    scale, h = 0.5, 1e-6
    r = A.backward_head(q, k, v, do, scale, keep=keep)
    f = r["fwd"]
    assert np.all(f["O"][3] == 0) and f["LSE"][3] == -np.inf
    assert np.all(r["dQ"][3] == 0)
    for which, an in ((0, r["dQ"]), (1, r["dK"]), (2, r["dV"])):
        args = [q, k, v]
        g = np.zeros_like(args[which])
        for idx in np.ndindex(g.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            g[idx] = (masked_loss(*plus, do, scale, keep) - masked_loss(*minus, do, scale, keep)) / (2 * h)
        assert np.all(np.abs(an - g) <= 1e-7 * np.abs(g).max() + 1e-9)


def test_torch_autograd_cross_check_block_mask():
    # a separately written formula: softmax over the kept scores (rows with
    # none kept give zero), through float64 autograd
    B, H, N, d = 1, 2, 300, 16
    q, k, v, do = (rnd(60 + t, B, H, N, d) for t in range(4))
    bm = np.random.default_rng(65).integers(0, 3, (3, 3))
    bm[1, :] = 0  # query tile 1 keeps nothing
    keep = A.block_mask_keep(bm, N)
    out = A.backward(q, k, v, do, 0.25, keep=keep)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    s = 0.25 * tq @ tk.transpose(-1, -2)
    km = torch.tensor(keep)
    s = s.masked_fill(~km, float("-inf"))
    row_any = km.any(-1, keepdim=True)
    p = torch.where(row_any, torch.softmax(torch.where(row_any, s, torch.zeros_like(s)), -1),
                    torch.zeros_like(s))
    p = torch.where(km, p, torch.zeros_like(p))
    o = p @ tv
    (o * torch.tensor(do)).sum().backward()
    assert rel(out["O"], o.detach().numpy()) <= 1e-12
    for name, g in (("dQ", tq.grad), ("dK", tk.grad), ("dV", tv.grad)):
        assert rel(out[name], g.numpy()) <= 1e-12
    assert np.all(out["LSE"][:, :, 128:256] == -np.inf)


# ---------------------------------------------------------------- MHA layer
def _torch_layer(x, w_qkv, w_o, dy, H):
    """The same layer through torch float64 autograd, written separately:
    heads split with view/transpose, softmax by torch, causal mask by tril."""
    x, w_qkv, w_o = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (x, w_qkv, w_o))
    B, N, C = x.shape
    d = C // H
    qkv = x @ w_qkv
    q, k, v = (qkv[..., c * C:(c + 1) * C].view(B, N, H, d).transpose(1, 2) for c in range(3))
    s = (q @ k.transpose(-1, -2)) / d ** 0.5
    s = s.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf"))
    o = torch.softmax(s, dim=-1) @ v
    y = o.transpose(1, 2).reshape(B, N, C) @ w_o
    (y * torch.tensor(dy)).sum().backward()
    return y.detach().numpy(), x.grad.numpy(), w_qkv.grad.numpy(), w_o.grad.numpy()


def test_mha_layer_against_torch_autograd():
    r = np.random.default_rng(11)
    B, N, H, d = 3, 10, 2, 4
    C = H * d
    x = r.standard_normal((B, N, C))
    w_qkv = r.standard_normal((C, 3 * C)) / np.sqrt(C)
    w_o = r.standard_normal((C, C)) / np.sqrt(C)
    dy = r.standard_normal((B, N, C))
    out = oracle.mha_layer(x, w_qkv, w_o, dy, H)
    y, dx, dwq, dwo = _torch_layer(x, w_qkv, w_o, dy, H)
    for name, ref in (("y", y), ("dx", dx), ("dW_qkv", dwq), ("dW_o", dwo)):
        np.testing.assert_allclose(out[name], ref, rtol=1e-11, atol=1e-12, err_msg=name)


def test_mha_layer_finite_differences():
    r = np.random.default_rng(12)
    B, N, H, d = 1, 5, 2, 3
    C = H * d
    x = r.standard_normal((B, N, C))
    w_qkv = r.standard_normal((C, 3 * C)) / np.sqrt(C)
    w_o = r.standard_normal((C, C)) / np.sqrt(C)
    dy = r.standard_normal((B, N, C))
    out = oracle.mha_layer(x, w_qkv, w_o, dy, H)

    def loss(x_, wq_, wo_):
        return float((oracle.mha_layer(x_, wq_, wo_, dy, H)["y"] * dy).sum())

    h = 1e-6
    for name, arr, idxs in (("dx", x, [(0, 0, 0), (0, 4, 5), (0, 2, 3)]),
                            ("dW_qkv", w_qkv, [(0, 0), (5, 17), (3, 8)]),
                            ("dW_o", w_o, [(0, 0), (5, 5), (2, 4)])):
        for ix in idxs:
            ap, am = arr.copy(), arr.copy()
            ap[ix] += h
            am[ix] -= h
            args_p = {"dx": (ap, w_qkv, w_o), "dW_qkv": (x, ap, w_o), "dW_o": (x, w_qkv, ap)}[name]
            args_m = {"dx": (am, w_qkv, w_o), "dW_qkv": (x, am, w_o), "dW_o": (x, w_qkv, am)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - out[name][ix]) <= 1e-6 * max(1.0, np.abs(out[name]).max()), (name, ix)


# ------------------------------------------------- backward-over-backward
def _bob_inputs(seed, n=7, d=3):
    r = np.random.default_rng(seed)
    return [r.standard_normal((n, d)) for _ in range(7)]


def _l2(q, k, v, do, uq, uk, uv, scale, causal):
    g = A.backward_head(q, k, v, do, scale, causal)
    return float((uq * g["dQ"]).sum() + (uk * g["dK"]).sum() + (uv * g["dV"]).sum())


@pytest.mark.parametrize("causal", [True, False])
def test_double_backward_finite_differences(causal):
    q, k, v, do, uq, uk, uv = _bob_inputs(21 + causal)
    scale = 0.6
    out = oracle.double_backward_head(q, k, v, do, uq, uk, uv, scale, causal)
    h = 1e-6
    args = [q, k, v, do]
    for idx, name in enumerate(("gQ", "gK", "gV", "gdO")):
        fd = np.zeros_like(args[idx])
        for ix in np.ndindex(*fd.shape):
            ap = [a.copy() for a in args]
            am = [a.copy() for a in args]
            ap[idx][ix] += h
            am[idx][ix] -= h
            fd[ix] = (_l2(*ap, uq, uk, uv, scale, causal) - _l2(*am, uq, uk, uv, scale, causal)) / (2 * h)
        err = np.abs(fd - out[name]).max()
        assert err <= 1e-7 * max(1.0, np.abs(out[name]).max()), (name, err)


def test_double_backward_against_torch_double_backward():
    q, k, v, do, uq, uk, uv = (torch.tensor(a) for a in _bob_inputs(23, n=9, d=4))
    scale = 0.5
    out = oracle.double_backward_head(*(t.numpy() for t in (q, k, v, do, uq, uk, uv)), scale, True)
    q, k, v, do = (t.clone().requires_grad_(True) for t in (q, k, v, do))
    n = q.shape[0]
    s = (q @ k.T) * scale
    s = s.masked_fill(~torch.ones(n, n, dtype=torch.bool).tril(), float("-inf"))
    o = torch.softmax(s, dim=-1) @ v
    dq, dk, dv = torch.autograd.grad(o, (q, k, v), do, create_graph=True)
    l2 = (uq * dq).sum() + (uk * dk).sum() + (uv * dv).sum()
    gq, gk, gv, gdo = torch.autograd.grad(l2, (q, k, v, do))
    for name, t in (("gQ", gq), ("gK", gk), ("gV", gv), ("gdO", gdo)):
        np.testing.assert_allclose(out[name], t.numpy(), rtol=1e-10, atol=1e-12, err_msg=name)


def test_double_backward_is_linear_in_the_cotangents():
    q, k, v, do, uq, uk, uv = _bob_inputs(24)
    a = oracle.double_backward_head(q, k, v, do, uq, uk, uv, 0.7)
    b = oracle.double_backward_head(q, k, v, do, 2 * uq, 2 * uk, 2 * uv, 0.7)
    z = oracle.double_backward_head(q, k, v, do, 0 * uq, 0 * uk, 0 * uv, 0.7)
    for name in ("gQ", "gK", "gV", "gdO"):
        np.testing.assert_allclose(b[name], 2 * a[name], rtol=1e-12, atol=1e-13)
        assert np.abs(z[name]).max() == 0.0


def test_double_backward_row_side_is_affine_in_the_two_row_scalars():
    # gQ and gdO of a row are fixed vectors combined with r and g (the
    # structure the FlashBoB listing states): accumulating the seven vectors
    # below, whose per-pair weights need neither scalar, and combining them
    # with r and g reproduces the oracle
    q, k, v, do, uq, uk, uv = _bob_inputs(25, n=11, d=5)
    scale, n = 0.45, 11
    out = oracle.double_backward_head(q, k, v, do, uq, uk, uv, scale, True)
    f = A.forward_head(q, k, v, scale, True)
    P = f["P"]
    dP = do @ v.T
    D = (P * dP).sum(axis=1, keepdims=True)
    M = scale * (uq @ k.T + q @ uk.T)
    W = do @ uv.T
    r = (P * M).sum(axis=1, keepdims=True)
    g = (P * M * dP).sum(axis=1, keepdims=True) - 2 * r * D + (P * W).sum(axis=1, keepdims=True)
    np.testing.assert_allclose(r[:, 0], out["r"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g[:, 0], out["g"], rtol=1e-12, atol=1e-13)
    x1 = (P * (dP - D)) @ uk
    x2 = (P * (M * (dP - D) + W)) @ k
    x3 = (P * dP) @ k
    x4 = P @ k
    y1, y2, y3 = (P * M) @ v, P @ v, P @ uv
    np.testing.assert_allclose(scale * (x1 + x2 - r * x3 - g * x4), out["gQ"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(y1 - r * y2 + y3, out["gdO"], rtol=1e-11, atol=1e-12)


def test_double_backward_single_position_closed_form():
    # N = 1: P = 1, so dS = E = dS2 = 0 and only dV = dO depends on dO:
    # gQ = gK = gV = 0, gdO = U_V
    r = np.random.default_rng(26)
    q, k, v, do, uq, uk, uv = (r.standard_normal((1, 6)) for _ in range(7))
    out = oracle.double_backward_head(q, k, v, do, uq, uk, uv, 0.8)
    for name in ("gQ", "gK", "gV"):
        assert np.abs(out[name]).max() == 0.0, name
    np.testing.assert_array_equal(out["gdO"], uv)
