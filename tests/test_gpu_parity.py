"""GPU parity: the CUDA library (through its C ABI) against the float64 oracle.

Small and medium shapes are compared element by element over every output,
and so are 8-head cases of 8,192 (d = 128) and 16,384 (d = 64) tokens, whose
key tiles walk 64 and 128 query tiles, through the oracle's row-blocked pass.
Of the 16,384-token x 32-head workload two whole heads are compared element by
element and two more on sampled rows and the last key rows; the 262,144-token
workload on sampled query rows and its last key rows (the only keys whose
gradients the oracle can form without a full head), plus identities that
hold at any size.

Tolerances (max |gpu - oracle| / max |oracle| per output): 1e-5 for the fp32
path, 2e-2 for the bf16 path (bf16 inputs and outputs, fp32 accumulation).
"""
import numpy as np
import pytest
import torch

import oracle
from seeded_inputs import CONFIGS, as_f64, block_mask, draw

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}


def rel(a, b, scale=None):
    """max |a - b| / max |b|. A reference that is identically zero (dQ and dK
    at N = 1) is measured against `scale`, the size of the other gradients."""
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    denom = np.abs(b).max()
    if denom == 0.0 and scale is not None:
        denom = scale
    return float(np.abs(a - b).max() / max(denom, 1e-30))


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import causal_softmax_attention_b200 as lib
    return lib


def run_gpu(csa, q, k, v, do, causal, scale):
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev).contiguous() for t in (q, k, v, do))
    o, lse = csa.forward(qd, kd, vd, causal, scale)
    dq, dk, dv = csa.backward(qd, kd, vd, o, dod, lse, causal, scale)
    torch.cuda.synchronize()
    assert csa.attn_fwd_last_status() == 0
    return {"O": o, "LSE": lse, "dQ": dq, "dK": dk, "dV": dv}


def compare_full(csa, B, H, N, d, dtype, seed, causal=True, qk_gain=1.0):
    q, k, v, do = draw(B, H, N, d, seed, dtype, qk_gain)
    scale = d ** -0.5
    g = run_gpu(csa, q, k, v, do, causal, scale)
    ref = oracle.backward(as_f64(q), as_f64(k), as_f64(v), as_f64(do), scale, causal)
    tol = TOL[dtype]
    gscale = max(np.abs(ref[n]).max() for n in ("dQ", "dK", "dV"))
    errs = {name: rel(as_f64(g[name].cpu()), ref[name], gscale) for name in ("O", "dQ", "dK", "dV")}
    lse_err = float(np.abs(as_f64(g["LSE"].cpu()) - ref["LSE"]).max())
    for name, e in errs.items():
        assert e <= tol, (name, e, errs)
    assert lse_err <= (1e-5 if dtype == "f32" else 1e-3), lse_err
    return errs


# ------------------------------------------------------------------ the configs
@pytest.mark.parametrize("name", ["c1", "c2_f32", "c2_bf16", "c3"])
def test_config_parity(csa, name):
    c = CONFIGS[name]
    compare_full(csa, c.B, c.H, c.N, c.d, c.dtype, c.seed, c.causal, c.qk_gain)


# ------------------------------------------------------------------ ragged / edge shapes
@pytest.mark.parametrize("B,H,N,d,causal", [
    (1, 2, 200, 64, True), (2, 1, 1000, 128, True), (1, 1, 1, 32, True),
    (1, 1, 130, 128, True), (1, 1, 127, 64, True), (1, 3, 384, 32, False),
    (2, 2, 257, 64, False), (1, 1, 129, 128, False), (3, 2, 640, 128, True),
])
def test_bf16_shapes(csa, B, H, N, d, causal):
    compare_full(csa, B, H, N, d, "bf16", 100 + N, causal)


@pytest.mark.parametrize("B,H,N,d,causal", [
    (1, 2, 100, 48, True), (1, 1, 1, 7, True), (2, 1, 70, 64, False), (1, 1, 300, 128, True),
    (2, 3, 33, 1, True),
])
def test_f32_shapes(csa, B, H, N, d, causal):
    compare_full(csa, B, H, N, d, "f32", 200 + N, causal)


# ------------------------------------------------------------------ properties on the GPU
@pytest.mark.parametrize("dtype,recompute", [("bf16", False), ("f32", False), ("bf16", True),
                                             ("f32", True)])
def test_backward_host_pipelined_matches_device(csa, dtype, recompute):
    # host buffers in and out, heads in groups on three streams: the same
    # gradients as one attn_bwd call on device buffers (dK, dV bit for bit;
    # dQ up to the order of its fp32 atomic sums); with the forward recomputed
    # on the device per group, O and LSE never cross from the host
    B, H, N, d = 2, 5, 300, 64
    q, k, v, do = draw(B, H, N, d, 77, dtype)
    g = run_gpu(csa, q, k, v, do, True, d ** -0.5)
    dev = torch.device("cuda")
    host = {n: t.pin_memory() for n, t in (("q", q), ("k", k), ("v", v), ("dout", do))}
    host["o"] = g["O"].cpu().pin_memory()
    host["lse"] = g["LSE"].cpu().pin_memory()
    outs = {n: torch.empty_like(host["q"]).pin_memory() for n in ("dq", "dk", "dv")}
    bufs = {n: torch.empty_like(host[n], device=dev) for n in ("q", "k", "v", "o", "dout", "lse")}
    bufs.update({n: torch.empty_like(bufs["q"]) for n in ("dq", "dk", "dv")})
    bufs["workspace"] = torch.empty(csa.chunk_workspace_bytes(B, H, N, d, bufs["q"].dtype, 4),
                                    dtype=torch.uint8, device=dev)
    csa.backward_host(host["q"], host["k"], host["v"], None if recompute else host["o"],
                      host["dout"], None if recompute else host["lse"],
                      outs["dq"], outs["dk"], outs["dv"], bufs, True, d ** -0.5, chunks=4,
                      recompute_forward=recompute)
    torch.cuda.synchronize()
    if recompute:
        assert torch.equal(bufs["o"], g["O"]) and torch.equal(bufs["lse"], g["LSE"])
    assert torch.equal(outs["dk"], g["dK"].cpu())
    assert torch.equal(outs["dv"], g["dV"].cpu())
    ref = as_f64(g["dQ"].cpu())
    assert rel(as_f64(outs["dq"]), ref, np.abs(ref).max()) <= (1e-6 if dtype == "f32" else 1e-2)


@pytest.mark.parametrize("d", [64, 128])
def test_running_max_raised_every_key_tile(csa, d):
    # Scores grow by more than 8 (log2 units) from one key tile to the next,
    # so the forward's running maximum is raised, and O rescaled in TMEM, on
    # every tile; O and LSE, and the dK and dV computed from them, must still
    # match. dQ is left out here: every key carries a large common component
    # (up to ~120 along u) that cancels in dQ_i = sum_j dS_ij K_j because each
    # row of dS sums to zero, and with dS rounded to bf16 for the MMA that
    # cancellation leaves a residue of a few percent of the small dQ, in any
    # bf16 backward. The other parity tests cover dQ.
    B, H, N = 1, 2, 5 * 128 + 37
    g = torch.Generator("cpu").manual_seed(91)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g) for _ in range(4))
    u = torch.randn(d, generator=g)
    u = u / u.norm()
    scale = d ** -0.5
    shift = 6.0 / scale / 2.0 * (torch.arange(N) // 128).float()  # q.k gains 2*shift
    q = q + 2.0 * u
    k = k + shift[:, None] * u
    q, k, v, do = (t.to(torch.bfloat16) for t in (q, k, v, do))
    gr = run_gpu(csa, q, k, v, do, True, scale)
    ref = oracle.backward(as_f64(q), as_f64(k), as_f64(v), as_f64(do), scale, True)
    gscale = max(np.abs(ref[n]).max() for n in ("dQ", "dK", "dV"))
    for name in ("O", "dK", "dV"):
        e = rel(as_f64(gr[name].cpu()), ref[name], None if name == "O" else gscale)
        assert e <= TOL["bf16"], (name, e)
    assert np.abs(as_f64(gr["LSE"].cpu()) - ref["LSE"]).max() <= 1e-3 * max(1.0, np.abs(ref["LSE"]).max())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("upper", [True, False])
def test_forward_key_halves_far_apart(csa, d, upper):
    # Inside every key tile the keys of one half (upper: local index >= 64)
    # score about 20 log2 units above the other half for every query. The
    # forward keeps a running maximum, sum and accumulator per half of each
    # tile's keys and combines them once with weights 2^(m_g - M); here one
    # half's weight is ~2^-20, and on the diagonal tile rows below 64 see
    # only the lower half of that tile but both halves of the earlier ones.
    B, H, N = 1, 2, 4 * 128 + 45
    g = torch.Generator("cpu").manual_seed(93 + d + int(upper))
    q, k, v, do = (torch.randn(B, H, N, d, generator=g) for _ in range(4))
    u = torch.randn(d, generator=g)
    u = u / u.norm()
    scale = d ** -0.5
    c = 20.0 / (scale * 2.0 * np.log2(np.e))  # q.k gains 2c: 20 log2 units
    half = (torch.arange(N) % 128) >= 64
    lift = half if upper else ~half
    q = q + 2.0 * u
    k = k + (c * lift.float())[:, None] * u
    q, k, v, do = (t.to(torch.bfloat16) for t in (q, k, v, do))
    gr = run_gpu(csa, q, k, v, do, True, scale)
    ref_o, ref_lse = oracle.forward(as_f64(q), as_f64(k), as_f64(v), scale, True)
    e = rel(as_f64(gr["O"].cpu()), ref_o, None)
    assert e <= TOL["bf16"], e
    assert np.abs(as_f64(gr["LSE"].cpu()) - ref_lse).max() <= 1e-3 * max(1.0, np.abs(ref_lse).max())


def run_masked(csa, q, k, v, do, bm, scale):
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev).contiguous() for t in (q, k, v, do))
    B, H, N, d = q.shape
    mask = torch.tensor(bm, dtype=torch.uint8, device=dev).contiguous()
    o = torch.empty_like(qd)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    csa.attn_fwd_masked(qd, kd, vd, o, lse, mask, scale)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    csa.attn_bwd_masked(qd, kd, vd, o, dod, lse, dq, dk, dv, mask, csa.new_workspace(qd), scale)
    torch.cuda.synchronize()
    assert csa.attn_fwd_last_status() == 0
    return {"O": o, "LSE": lse, "dQ": dq, "dK": dk, "dV": dv}


def compare_masked(csa, B, H, N, d, bm, seed):
    q, k, v, do = draw(B, H, N, d, seed, "bf16")
    scale = d ** -0.5
    g = run_masked(csa, q, k, v, do, bm, scale)
    keep = oracle.block_mask_keep(bm, N)
    ref = oracle.backward(as_f64(q), as_f64(k), as_f64(v), as_f64(do), scale, keep=keep)
    gscale = max(np.abs(ref[n]).max() for n in ("dQ", "dK", "dV"))
    for name in ("O", "dQ", "dK", "dV"):
        e = rel(as_f64(g[name].cpu()), ref[name], gscale if name != "O" else None)
        assert e <= TOL["bf16"], (name, e)
    lse = as_f64(g["LSE"].cpu())
    empty = np.isneginf(ref["LSE"])
    assert np.array_equal(np.isneginf(lse), empty)
    assert np.abs(lse[~empty] - ref["LSE"][~empty]).max() <= 1e-3
    return g, ref


@pytest.mark.parametrize("d", [32, 64, 128])
def test_block_sparse_parity(csa, d):
    # kinds 0 / 1 / 2 anywhere, an empty query tile (O = 0, LSE = -inf), a
    # key tile no query meets (dK = dV = 0), kind 2 off the diagonal
    N = 5 * 128 + 23
    bm = np.random.default_rng(d).integers(0, 3, (6, 6))
    bm[2, :] = 0
    bm[:, 4] = 0
    bm[5, 1] = 2
    g, ref = compare_masked(csa, 1, 2, N, d, bm, 300 + d)
    assert torch.all(g["O"][:, :, 256:384] == 0)
    assert torch.all(g["dQ"][:, :, 256:384] == 0)
    assert torch.all(g["dK"][:, :, 512:640] == 0) and torch.all(g["dV"][:, :, 512:640] == 0)


def test_block_sparse_sliding_window(csa):
    # local attention: each query tile sees its own tile (causally) and the
    # two before it
    N, w = 8 * 128, 2
    t = np.arange(8)
    bm = np.where(t[:, None] == t[None, :], 2,
                  np.where((t[None, :] < t[:, None]) & (t[None, :] >= t[:, None] - w), 1, 0))
    compare_masked(csa, 2, 2, N, 64, bm, 321)


def test_causal_block_mask_matches_the_causal_path(csa):
    B, H, N, d = 1, 3, 3 * 128 + 50, 128
    q, k, v, do = draw(B, H, N, d, 333, "bf16")
    t = np.arange(-(-N // 128))
    bm = np.where(t[:, None] > t[None, :], 1, np.where(t[:, None] == t[None, :], 2, 0))
    gm = run_masked(csa, q, k, v, do, bm, d ** -0.5)
    gc = run_gpu(csa, q, k, v, do, True, d ** -0.5)
    for name in ("O", "LSE", "dK", "dV"):
        assert torch.equal(gm[name], gc[name]), name
    ref = as_f64(gc["dQ"].cpu())
    assert rel(as_f64(gm["dQ"].cpu()), ref, np.abs(ref).max()) <= 1e-2


def test_block_mask_longer_than_the_shared_bitmaps(csa):
    # d = 128 keeps a key tile's column in shared memory only up to 2,560
    # tiles; past that the kernels walk the mask in global memory. Under a
    # two-tile window, query tile t sees key tiles t-1 and t, so the three
    # tiles t-1 .. t+1 hold every score that O, LSE, dQ of query tile t and
    # dK, dV of key tile t depend on: the oracle runs on those 384 positions.
    B, H, d = 1, 1, 128
    T = 2600
    N = T * 128 - 77
    q, k, v, do = draw(B, H, N, d, 351, "bf16")
    bm = block_mask("window:2", N)
    g = run_masked(csa, q, k, v, do, bm, d ** -0.5)
    local_bm = block_mask("window:2", 3 * 128)
    for t in (1, 1300, T - 2):
        lo, hi = 128 * (t - 1), min(N, 128 * (t + 2))
        sl = [as_f64(x[0, 0, lo:hi]) for x in (q, k, v, do)]
        keep = oracle.block_mask_keep(local_bm[: -(-(hi - lo) // 128), : -(-(hi - lo) // 128)], hi - lo)
        ref = oracle.backward(*(x[None, None] for x in sl), d ** -0.5, keep=keep)
        a, b = 128, min(256, hi - lo)
        gscale = max(np.abs(ref[n][0, 0, a:b]).max() for n in ("dQ", "dK", "dV"))
        for name in ("O", "dQ", "dK", "dV"):
            got = as_f64(g[name][0, 0, lo + a:lo + b].cpu())
            e = rel(got, ref[name][0, 0, a:b], gscale if name != "O" else None)
            assert e <= TOL["bf16"], (t, name, e)
        lse = as_f64(g["LSE"][0, 0, lo + a:lo + b].cpu())
        assert np.abs(lse - ref["LSE"][0, 0, a:b]).max() <= 1e-3, t


def test_staged_masked_backward_matches_the_single_call(csa):
    # attn_bwd_preprocess + attn_bwd_main_masked + attn_bwd_dq_convert is
    # attn_bwd_masked; the window mask comes from the bench's mask recipe
    B, H, N, d = 1, 2, 6 * 128 + 40, 64
    q, k, v, do = draw(B, H, N, d, 341, "bf16")
    bm = block_mask("window:3", N)
    g = run_masked(csa, q, k, v, do, bm, d ** -0.5)
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    mask = torch.from_numpy(bm).to(dev)
    ws = csa.new_workspace(qd)
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    csa.attn_bwd_preprocess(g["O"], dod, g["LSE"], ws)
    csa.attn_bwd_main_masked(qd, kd, vd, dod, dq, dk, dv, mask, ws)
    csa.attn_bwd_dq_convert(dq, ws)
    torch.cuda.synchronize()
    assert csa.attn_last_status(ws) == 0
    assert torch.equal(dk, g["dK"]) and torch.equal(dv, g["dV"])
    ref = as_f64(g["dQ"].cpu())
    assert rel(as_f64(dq.cpu()), ref, np.abs(ref).max()) <= 1e-2


def run_strided(csa, q, k, v, do, causal, scale, layout):
    """Forward and backward through the strided entry points, the tensors
    held in `layout`: "bnhd" ([B, N, H, d] arrays) or "packed" (q, k, v in
    one [B, N, 3, H, d] array and dq, dk, dv in another; o, dO [B, N, H, d])."""
    dev = torch.device("cuda")
    B, H, N, d = q.shape

    def bnhd(x):  # a [B, N, H, d] array holding x, returned as its [B, H, N, d] view
        return x.to(dev).permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)

    if layout == "packed":
        qkv = torch.stack([x.to(dev).permute(0, 2, 1, 3) for x in (q, k, v)], dim=2).contiguous()
        qv, kv, vv = (qkv[:, :, c].permute(0, 2, 1, 3) for c in range(3))
        dqkv = torch.full_like(qkv, float("nan"))
        dq, dk, dv = (dqkv[:, :, c].permute(0, 2, 1, 3) for c in range(3))
    else:
        qv, kv, vv = bnhd(q), bnhd(k), bnhd(v)
        dq, dk, dv = (bnhd(torch.full_like(q, float("nan"))) for _ in range(3))
    dov = bnhd(do)
    o = bnhd(torch.full_like(q, float("nan")))
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    csa.attn_fwd_strided(qv, kv, vv, o, lse, causal, scale)
    csa.attn_bwd_strided(qv, kv, vv, o, dov, lse, dq, dk, dv, csa.new_workspace(qv.contiguous()),
                         causal, scale)
    torch.cuda.synchronize()
    assert csa.attn_fwd_last_status() == 0
    return {"O": o, "LSE": lse, "dQ": dq, "dK": dk, "dV": dv}


@pytest.mark.parametrize("dtype,d,layout", [("bf16", 64, "bnhd"), ("bf16", 128, "bnhd"),
                                            ("bf16", 64, "packed"), ("bf16", 32, "packed"),
                                            ("bf16", 128, "packed"),
                                            ("f32", 48, "bnhd"), ("f32", 7, "packed")])
def test_strided_layouts_match_the_contiguous_path(csa, dtype, d, layout):
    # the same kernels on the same values: O, LSE, dK, dV bit-identical to the
    # contiguous path (dQ too for f32; bf16 dQ sums in atomic order)
    B, H, N = 2, 3, 2 * 128 + 45
    q, k, v, do = draw(B, H, N, d, 361 + d, dtype)
    c = run_gpu(csa, q, k, v, do, True, d ** -0.5)
    g = run_strided(csa, q, k, v, do, True, d ** -0.5, layout)
    for name in ("O", "LSE", "dK", "dV") + (("dQ",) if dtype == "f32" else ()):
        assert torch.equal(g[name].contiguous(), c[name]), name
    if dtype == "bf16":
        ref = as_f64(c["dQ"].cpu())
        assert rel(as_f64(g["dQ"].cpu()), ref) <= 1e-2


def test_strided_ddx_issue217_tables_against_the_oracle(csa):
    # the repro's (seq, pos, head, channel) tables consumed in place (f32,
    # 4 channels), against the oracle on the same values; loss 1/2 sum O^2
    # so dO = O
    from seeded_inputs import ddx_issue217_input
    S, T, H, C = 3, 8, 2, 4
    # [B, H, N, d], rounded to the fp32 values the GPU receives
    qh, kh, vh = (x.astype(np.float32).astype(np.float64) for x in ddx_issue217_input(S, T, H, C))
    scale = 1.0 / 2.0
    o_ref, _ = oracle.forward(qh, kh, vh, scale, True)
    ref = oracle.backward(qh, kh, vh, o_ref, scale, True)
    dev = torch.device("cuda")

    def table(x):  # [S, T, H, C] float32 table, viewed as [B, H, N, d]
        return torch.from_numpy(x).float().to(dev).permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)

    q, k, v = table(qh), table(kh), table(vh)
    o = table(np.zeros_like(qh))
    lse = torch.empty(S, H, T, dtype=torch.float32, device=dev)
    csa.attn_fwd_strided(q, k, v, o, lse, True, scale)
    dout = o.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    dq, dk, dv = (table(np.zeros_like(qh)) for _ in range(3))
    csa.attn_bwd_strided(q, k, v, o, dout, lse, dq, dk, dv, csa.new_workspace(q.contiguous()),
                         True, scale)
    torch.cuda.synchronize()
    assert rel(as_f64(o.cpu()), o_ref) <= 1e-5
    gscale = max(np.abs(ref[n]).max() for n in ("dQ", "dK", "dV"))
    for name, t in (("dQ", dq), ("dK", dk), ("dV", dv)):
        assert rel(as_f64(t.cpu()), ref[name], gscale) <= 1e-5, name


@pytest.mark.parametrize("B,N,C,H", [(12, 64, 128, 4), (2, 1000, 512, 4), (1, 700, 1024, 8)])
def test_mha_layer_step_against_the_oracle(csa, B, N, C, H):
    # the first shape is ddx issue #217's nanoGPT-shaped layer (batch 12,
    # 64 positions, 128 channels, 4 heads); bf16 storage between the steps
    from causal_softmax_attention_b200 import layer
    from seeded_inputs import draw_layer
    x, w_qkv, w_o, dy = draw_layer(B, N, C, 400 + C)
    ref = oracle.mha_layer(as_f64(x), as_f64(w_qkv), as_f64(w_o), as_f64(dy), H)
    dev = torch.device("cuda")
    xd, wq, wo, dyd = (t.to(dev) for t in (x, w_qkv, w_o, dy))
    y, saved = layer.layer_forward(xd, wq, wo, H)
    dx, dwq, dwo = layer.layer_backward(dyd, saved, wq, wo, H)
    torch.cuda.synchronize()
    assert csa.attn_fwd_last_status() == 0
    for name, got in (("y", y), ("dx", dx), ("dW_qkv", dwq), ("dW_o", dwo)):
        e = rel(as_f64(got.cpu()), ref[name])
        assert e <= TOL["bf16"], (name, e)


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 1, 256, 64, True), (2, 3, 200, 48, True),
                                             (2, 3, 200, 48, False), (1, 2, 130, 128, True),
                                             (3, 1, 77, 7, True), (1, 1, 1, 32, True)])
def test_double_backward_against_the_oracle(csa, B, H, N, d, causal):
    q, k, v, do = draw(B, H, N, d, 500 + N, "f32")
    uq, uk, uv, _ = draw(B, H, N, d, 600 + N, "f32")
    scale = d ** -0.5
    ref = oracle.double_backward(*(as_f64(t) for t in (q, k, v, do, uq, uk, uv)), scale, causal)
    dev = torch.device("cuda")
    qd, kd, vd, dod, uqd, ukd, uvd = (t.to(dev) for t in (q, k, v, do, uq, uk, uv))
    o, lse = csa.forward(qd, kd, vd, causal, scale)
    gq, gk, gv, gdo = csa.backward_over_backward(qd, kd, vd, o, dod, lse, uqd, ukd, uvd, causal,
                                                 scale)
    torch.cuda.synchronize()
    gscale = max(np.abs(ref[n]).max() for n in ("gQ", "gK", "gV", "gdO"))
    for name, t in (("gQ", gq), ("gK", gk), ("gV", gv), ("gdO", gdo)):
        assert rel(as_f64(t.cpu()), ref[name], gscale) <= TOL["f32"], name


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 2, 2100, 64, True), (1, 1, 2048 + 77, 128, True),
                                             (2, 1, 300, 32, True), (1, 1, 1100, 32, True),
                                             (1, 2, 700, 64, False), (2, 3, 260, 64, False),
                                             (2, 2, 129, 128, False), (1, 1, 1, 64, True)])
def test_double_backward_bf16_against_the_oracle(csa, B, H, N, d, causal):
    # the tensor-core kernels: 2,100 and 2,125 tokens walk 17 tiles (key tile
    # 0 meets every query tile), 1,100 at d = 32 nine (three score sets in both
    # sweeps); N = 1 has the closed form gQ = gK = gV = 0, gdO = U_V. The
    # oracle takes the bf16-rounded inputs widened to float64.
    q, k, v, do = draw(B, H, N, d, 800 + N, "bf16")
    uq, uk, uv, _ = draw(B, H, N, d, 850 + N, "bf16")
    scale = d ** -0.5
    ref = oracle.double_backward(*(as_f64(t) for t in (q, k, v, do, uq, uk, uv)), scale, causal)
    dev = torch.device("cuda")
    qd, kd, vd, dod, uqd, ukd, uvd = (t.to(dev) for t in (q, k, v, do, uq, uk, uv))
    o, lse = csa.forward(qd, kd, vd, causal, scale)
    outs = [torch.full_like(qd, float("nan")) for _ in range(4)]
    ws = torch.empty(csa.library().attn_bwd_bwd_workspace_bytes(B, H, N, d, csa.ATTN_BF16),
                     dtype=torch.uint8, device=dev)
    csa.attn_bwd_bwd(qd, kd, vd, o, dod, lse, uqd, ukd, uvd, *outs, ws, causal, scale)
    torch.cuda.synchronize()
    assert csa.attn_last_status(ws) == csa.ATTN_OK
    gscale = max(np.abs(ref[n]).max() for n in ("gQ", "gK", "gV", "gdO"))
    for name, t in zip(("gQ", "gK", "gV", "gdO"), outs):
        assert rel(as_f64(t.cpu()), ref[name], gscale) <= TOL["bf16"], name


@pytest.mark.parametrize("d", [64, 128])
def test_double_backward_timeout_is_reported(csa, d):
    # the armed one-shot fault withholds the rows kernel's first score
    # quarter: every bounded wait of both issuers, the TMA warp and the
    # element-wise warps ends, the status word says so, and the next call is
    # unaffected
    B, H, N = 1, 1, 300
    q, k, v, do = draw(B, H, N, d, 860 + d, "bf16")
    uq, uk, uv, _ = draw(B, H, N, d, 870 + d, "bf16")
    dev = torch.device("cuda")
    qd, kd, vd, dod, uqd, ukd, uvd = (t.to(dev) for t in (q, k, v, do, uq, uk, uv))
    o, lse = csa.forward(qd, kd, vd, True, d ** -0.5)
    ws = torch.empty(csa.library().attn_bwd_bwd_workspace_bytes(B, H, N, d, csa.ATTN_BF16),
                     dtype=torch.uint8, device=dev)
    outs = [torch.empty_like(qd) for _ in range(4)]
    assert csa.attn_test_arm_timeout(50_000_000) == csa.ATTN_OK
    csa.attn_bwd_bwd(qd, kd, vd, o, dod, lse, uqd, ukd, uvd, *outs, ws, True, d ** -0.5)
    torch.cuda.synchronize()
    assert csa.attn_last_status(ws) == csa.ATTN_ERR_TIMEOUT
    csa.attn_bwd_bwd(qd, kd, vd, o, dod, lse, uqd, ukd, uvd, *outs, ws, True, d ** -0.5)
    torch.cuda.synchronize()
    assert csa.attn_last_status(ws) == csa.ATTN_OK
    ref = oracle.double_backward(*(as_f64(t) for t in (q, k, v, do, uq, uk, uv)), d ** -0.5, True)
    gscale = max(np.abs(ref[n]).max() for n in ("gQ", "gK", "gV", "gdO"))
    for name, t in zip(("gQ", "gK", "gV", "gdO"), outs):
        assert rel(as_f64(t.cpu()), ref[name], gscale) <= TOL["bf16"], name


def test_forward_exponential_polynomial(csa):
    # the forward computes one exponential in four on the FMA pipe (Cody-Waite
    # reduction, degree-3 polynomial): against exact 2^x and against MUFU's
    # ex2.approx over the arguments the forward produces (<= 8: the running
    # maximum is raised once a score exceeds it by 8), the masked -inf
    # included; below -125 the polynomial clamps to 2^-125
    x = np.concatenate([np.linspace(-130.0, 8.0, 1 << 20), np.linspace(-1.0, 1.0, 4097),
                        [-np.inf, -125.5, -125.0, -124.99, -0.5, 0.5, -1e-30, 0.0, 8.0]])
    x = x.astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    poly, mufu = torch.empty_like(xd), torch.empty_like(xd)
    st = csa.library().attn_test_exp2(xd.data_ptr(), poly.data_ptr(), mufu.data_ptr(), x.size,
                                      torch.cuda.current_stream().cuda_stream)
    assert st == csa.ATTN_OK
    torch.cuda.synchronize()
    poly, mufu = poly.cpu().numpy().astype(np.float64), mufu.cpu().numpy().astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    inside = x >= -125.0
    assert np.all(np.isfinite(poly)) and np.all(poly >= 0.0)
    assert np.abs(poly[inside] / exact[inside] - 1.0).max() <= 1e-4
    assert np.all(poly[~inside] <= 2.0 ** -124)
    normal = x >= -126.0
    assert np.abs(mufu[normal] / exact[normal] - 1.0).max() <= 1e-6
    assert np.abs(poly[inside] / mufu[inside] - 1.0).max() <= 1.1e-4


def test_linearity_and_causality(csa):
    B, H, N, d = 1, 2, 768, 64
    q, k, v, do = draw(B, H, N, d, 7, "bf16")
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = csa.forward(qd, kd, vd)
    g1 = csa.backward(qd, kd, vd, o, dod, lse)
    g2 = csa.backward(qd, kd, vd, o, 2 * dod, lse)  # exact in bf16
    for a, b in zip(g1, g2):
        assert rel(as_f64(b.cpu()), 2 * as_f64(a.cpu())) <= 2e-2
    i0 = 300
    do0 = dod.clone()
    do0[:, :, i0:] = 0
    dq, dk, dv = csa.backward(qd, kd, vd, o, do0, lse)
    assert torch.count_nonzero(dq[:, :, i0:]) == 0
    assert torch.count_nonzero(dk[:, :, i0:]) == 0
    assert torch.count_nonzero(dv[:, :, i0:]) == 0
    # permuting heads permutes the outputs
    perm = [1, 0]
    op, lp = csa.forward(qd[:, perm].contiguous(), kd[:, perm].contiguous(), vd[:, perm].contiguous())
    assert torch.equal(op, o[:, perm])
    assert torch.equal(lp, lse[:, perm])


@pytest.mark.parametrize("d", [32, 64, 128])
def test_timeout_is_reported_and_context_survives(csa, d):
    # every d: one MMA issuer at d <= 64, two at d = 128; each side's bounded
    # waits must end once the first score tile never arrives
    B, H, N = 1, 1, 256
    q, k, v, do = draw(B, H, N, d, 9, "bf16")
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = csa.forward(qd, kd, vd)
    ws = csa.new_workspace(qd)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    assert csa.attn_test_arm_timeout(50_000_000) == csa.ATTN_OK  # ~25 ms of SM cycles
    csa.attn_bwd(qd, kd, vd, o, dod, lse, dq, dk, dv, ws)
    assert csa.attn_last_status(ws) == csa.ATTN_ERR_TIMEOUT
    # the next call is unaffected
    csa.attn_bwd(qd, kd, vd, o, dod, lse, dq, dk, dv, ws)
    assert csa.attn_last_status(ws) == csa.ATTN_OK
    ref = oracle.backward(as_f64(q), as_f64(k), as_f64(v), as_f64(do), d ** -0.5, True)
    assert rel(as_f64(dq.cpu()), ref["dQ"]) <= 2e-2


def test_nonfinite_inputs_propagate(csa):
    B, H, N, d = 1, 1, 256, 64
    q, k, v, do = draw(B, H, N, d, 11, "bf16")
    v[0, 0, 5, 3] = float("nan")
    g = run_gpu(csa, q, k, v, do, True, d ** -0.5)
    # row 5 of V reaches every O row that keeps key 5 (IEEE 0 * NaN may also
    # reach the masked rows of the same tile; no claim is made about those)
    assert torch.isnan(g["O"][0, 0, 5:, 3]).all()
    assert not torch.isnan(g["O"][0, 0, :, :3]).any()


# ------------------------------------------------------------------ long tile walks, every element
def full_head_parity(g, q, k, v, do, scale, heads, tol=TOL["bf16"]):
    """Every element of O, LSE, dQ, dK, dV of the given heads against the
    oracle's row-blocked pass over all query rows (the materialised head's
    result, without an N x N table); per head, gradients are measured
    against the largest of its three gradients, as in compare_full."""
    for (b, h) in heads:
        qh, kh, vh, doh = (as_f64(t[b, h]) for t in (q, k, v, do))
        ref = oracle.backward_blocked(qh, kh, vh, doh, scale, True)
        gscale = max(np.abs(ref[n]).max() for n in ("dQ", "dK", "dV"))
        for name in ("O", "dQ", "dK", "dV"):
            got = as_f64(g[name][b, h].cpu())
            e = rel(got, ref[name], None if name == "O" else gscale)
            assert e <= tol, ((b, h), name, e)
        assert np.abs(as_f64(g["LSE"][b, h].cpu()) - ref["LSE"]).max() <= 1e-3, (b, h)


@pytest.mark.parametrize("N,d,qk_gain", [(8192, 128, 1.0), (16384, 64, 0.5)])
def test_long_walk_every_element(csa, N, d, qk_gain):
    # 8 heads: key tile 0 accumulates dK, dV over 64 (d = 128) or 128 (d = 64)
    # query tiles in tensor memory, and the CTAs run in two L2 head groups of
    # unequal size (5 + 3 heads); every output element of every head is checked
    B, H = 1, 8
    q, k, v, do = draw(B, H, N, d, 700 + d, "bf16", qk_gain)
    g = run_gpu(csa, q, k, v, do, True, d ** -0.5)
    full_head_parity(g, q, k, v, do, d ** -0.5, [(0, h) for h in range(H)])


@pytest.mark.parametrize("world", [2, 3, 4])
def test_head_sharded_backward_against_the_oracle(csa, world):
    # every rank's block through shard.backward_shard, all ranks in this one
    # process writing into shared full-size gradients (6 heads: 3 + 3, 2 + 2
    # + 2, and 2 + 2 + 2 + none)
    from causal_softmax_attention_b200.shard import backward_shard, head_range
    B, H, N, d = 2, 3, 500, 64
    q, k, v, do = draw(B, H, N, d, 720 + world, "bf16")
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = csa.forward(qd, kd, vd, True, d ** -0.5)
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    covered = []
    for rank in range(world):
        start, end = head_range(B * H, world, rank)
        ws = torch.empty(max(1, csa.attn_bwd_workspace_bytes(1, max(1, end - start), N, d,
                                                                 qd.dtype)),
                         dtype=torch.uint8, device=dev)
        got = backward_shard(qd, kd, vd, o, dod, lse, dq, dk, dv, ws, world, rank, True,
                             d ** -0.5)
        assert got == (start, end)
        covered += list(range(start, end))
    torch.cuda.synchronize()
    assert covered == list(range(B * H))
    ref = oracle.backward(as_f64(q), as_f64(k), as_f64(v), as_f64(do), d ** -0.5, True)
    gscale = max(np.abs(ref[n]).max() for n in ("dQ", "dK", "dV"))
    for name, t in (("dQ", dq), ("dK", dk), ("dV", dv)):
        assert rel(as_f64(t.cpu()), ref[name], gscale) <= TOL["bf16"], name


@pytest.mark.parametrize("dtype,N,d", [("bf16", 333, 64), ("bf16", 130, 128), ("f32", 201, 48)])
def test_outputs_stay_inside_their_buffers(csa, dtype, N, d):
    # dQ, dK, dV (and O, LSE) written into the middle of larger buffers whose
    # guard regions hold a canary pattern: no byte outside the outputs changes
    B, H = 2, 2
    q, k, v, do = draw(B, H, N, d, 730 + N, dtype)
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    n = B * H * N * d
    guard = 4096  # elements on each side (a multiple of 8: keeps 16-byte alignment)

    def guarded(count, dt):
        buf = torch.empty(count + 2 * guard, dtype=dt, device=dev)
        buf.view(torch.uint8).fill_(0xA5)
        return buf

    bufs = {name: guarded(n, qd.dtype) for name in ("o", "dq", "dk", "dv")}
    bufs["lse"] = guarded(B * H * N, torch.float32)
    view = {name: b[guard:guard + n].view(B, H, N, d) for name, b in bufs.items() if name != "lse"}
    lse = bufs["lse"][guard:guard + B * H * N].view(B, H, N)
    csa.attn_fwd(qd, kd, vd, view["o"], lse, True, d ** -0.5)
    csa.attn_bwd(qd, kd, vd, view["o"], dod, lse, view["dq"], view["dk"], view["dv"],
                 csa.new_workspace(qd), True, d ** -0.5)
    torch.cuda.synchronize()
    for name, b in bufs.items():
        raw = b.view(torch.uint8)
        per = b.element_size()
        assert bool((raw[:guard * per] == 0xA5).all()), (name, "before")
        assert bool((raw[-guard * per:] == 0xA5).all()), (name, "after")
    ref = oracle.backward(as_f64(q), as_f64(k), as_f64(v), as_f64(do), d ** -0.5, True)
    gscale = max(np.abs(ref[n_]).max() for n_ in ("dQ", "dK", "dV"))
    for name in ("dq", "dk", "dv"):
        assert rel(as_f64(view[name].cpu()), ref["d" + name[1:].upper()], gscale) <= TOL[dtype]


# ------------------------------------------------------------------ N_q != N_k
def run_rect(csa, q, k, v, do, off, causal, scale):
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev).contiguous() for t in (q, k, v, do))
    o, lse = csa.forward_rect(qd, kd, vd, off, causal, scale)
    dq, dk, dv = csa.backward_rect(qd, kd, vd, o, dod, lse, off, causal, scale)
    torch.cuda.synchronize()
    assert csa.attn_fwd_last_status() == 0
    return {"O": o, "LSE": lse, "dQ": dq, "dK": dk, "dV": dv}


@pytest.mark.parametrize("dtype,nq,nk,off,causal,d", [
    ("bf16", 300, 1000, 700, True, 64),    # the KV-cache shape: the last 300 positions
    ("bf16", 200, 900, 333, True, 128),    # an offset off the tile grid: partial diagonal tiles
    ("bf16", 1000, 300, 0, True, 128),     # more queries than keys: rows past 300 see every key
    ("bf16", 257, 641, 50, True, 32),
    ("bf16", 200, 700, 0, False, 64),      # full attention, rectangular
    ("bf16", 700, 130, 0, False, 128),
    ("bf16", 129, 128, 5000, True, 64),    # every query after every key: the causal filter keeps all
    ("f32", 100, 333, 233, True, 48),
    ("f32", 333, 100, 0, True, 64),
    ("f32", 90, 200, 17, False, 7),
    ("f32", 70, 300, 101, True, 128),
    ("bf16", 300, 40, 0, False, 64),       # 40 keys: the forward's second softmax group sees none
    ("bf16", 100, 40, 20, True, 128),      # ... and, causal, rows before key 40 see fewer
])
def test_rectangular_against_the_oracle(csa, dtype, nq, nk, off, causal, d):
    from seeded_inputs import draw_rect
    B, H = 2, 3
    q, k, v, do = draw_rect(B, H, nq, nk, d, 900 + nq + nk, dtype)
    scale = d ** -0.5
    g = run_rect(csa, q, k, v, do, off, causal, scale)
    ref = oracle.backward(as_f64(q), as_f64(k), as_f64(v), as_f64(do), scale, causal, q_offset=off)
    gscale = max(np.abs(ref[n]).max() for n in ("dQ", "dK", "dV"))
    for name in ("O", "dQ", "dK", "dV"):
        e = rel(as_f64(g[name].cpu()), ref[name], None if name == "O" else gscale)
        assert e <= TOL[dtype], (name, e)
    assert np.abs(as_f64(g["LSE"].cpu()) - ref["LSE"]).max() <= (1e-5 if dtype == "f32" else 1e-3)
    if causal and off + nq < nk:
        # keys after the last query's position get no gradient
        assert torch.count_nonzero(g["dK"][:, :, off + nq:]) == 0
        assert torch.count_nonzero(g["dV"][:, :, off + nq:]) == 0


@pytest.mark.parametrize("d", [64, 128])
def test_rectangular_square_offset_zero_is_the_square_path(csa, d):
    # N_q == N_k with offset 0 runs the same kernels as attn_fwd / attn_bwd
    B, H, N = 1, 2, 3 * 128 + 11
    q, k, v, do = draw(B, H, N, d, 950 + d, "bf16")
    a = run_rect(csa, q, k, v, do, 0, True, d ** -0.5)
    b = run_gpu(csa, q, k, v, do, True, d ** -0.5)
    for name in ("O", "LSE", "dK", "dV"):
        assert torch.equal(a[name], b[name]), name
    ref = as_f64(b["dQ"].cpu())
    assert rel(as_f64(a["dQ"].cpu()), ref) <= 1e-2


def test_rectangular_rows_of_a_square_problem(csa):
    # the last 500 query rows of an 1800-token head with offset 1300: O, LSE
    # and dQ equal those rows of the square call (same kernels, same tiles
    # apart from the query tiles' alignment), within the bf16 tolerance
    B, H, N, nq, d = 1, 2, 1800, 500, 64
    q, k, v, do = draw(B, H, N, d, 960, "bf16")
    sq = run_gpu(csa, q, k, v, do, True, d ** -0.5)
    r = run_rect(csa, q[:, :, N - nq:].contiguous(), k, v, do[:, :, N - nq:].contiguous(),
                 N - nq, True, d ** -0.5)
    for name in ("O", "dQ"):
        ref = as_f64(sq[name][:, :, N - nq:].cpu())
        assert rel(as_f64(r[name].cpu()), ref) <= 2e-2, name
    assert np.abs(as_f64(r["LSE"].cpu()) - as_f64(sq["LSE"][:, :, N - nq:].cpu())).max() <= 1e-3


# ------------------------------------------------------------------ full-size workloads
def sampled_parity(csa, name, heads, n_rows=24, tail=128, full_heads=()):
    c = CONFIGS[name]
    q, k, v, do = draw(c.B, c.H, c.N, c.d, c.seed, c.dtype, c.qk_gain)
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    g = run_gpu(csa, q, k, v, do, True, c.scale)
    peak = torch.cuda.max_memory_allocated() - base
    # memory is linear in N: inputs, outputs and workspace are O(B*H*N*d)
    elems = c.B * c.H * c.N * c.d
    assert peak <= elems * 2 * 12 + c.B * c.H * c.N * 64, peak
    # whole heads, every element (every key tile's walk, the longest included)
    full_head_parity(g, q, k, v, do, c.scale, full_heads)
    rng = np.random.default_rng(c.seed)
    for (b, h) in heads:
        rows = np.sort(np.concatenate([rng.choice(c.N, n_rows - 4, replace=False),
                                       [0, 1, c.N // 2, c.N - 1]]))
        qh, kh, vh, doh = (as_f64(t[b, h]) for t in (q, k, v, do))
        r = oracle.query_rows(qh, kh, vh, doh, c.scale, rows, True)
        gq = as_f64(g["dQ"][b, h].cpu())[rows]
        assert rel(gq, r["dQ"]) <= TOL[c.dtype]
        assert rel(as_f64(g["O"][b, h].cpu())[rows], r["O"]) <= TOL[c.dtype]
        assert np.abs(as_f64(g["LSE"][b, h].cpu())[rows] - r["LSE"]).max() <= 1e-3
        t = oracle.key_tail(qh, kh, vh, doh, c.scale, c.N - tail, rows_per_block=256)
        assert rel(as_f64(g["dK"][b, h].cpu())[-tail:], t["dK"]) <= TOL[c.dtype]
        assert rel(as_f64(g["dV"][b, h].cpu())[-tail:], t["dV"]) <= TOL[c.dtype]
    # identities over all positions: sum_j dK_j = 0, sum_j dV_j = sum_i dO_i
    dk = g["dK"].double()
    dv = g["dV"].double()
    dod = do.to(dk.device).double()
    assert (dk.sum(2).abs() <= 1e-2 * dk.abs().sum(2) + 1e-6).all()
    assert ((dv.sum(2) - dod.sum(2)).abs() <= 1e-2 * dod.abs().sum(2) + 1e-3).all()
    for t in g.values():
        assert torch.isfinite(t).all()


def test_long_sequence_16k_parity(csa):
    # two whole heads element by element (their key tile 0 walks all 128
    # query tiles), sampled rows and the key tail of two more
    sampled_parity(csa, "c4", heads=[(0, 7), (1, 8)], full_heads=[(0, 0), (1, 15)])


def test_long_sequence_262k_parity(csa):
    # sampled dQ rows, and dK / dV of the last 2,048 keys (their 2,048 query
    # rows, each over all its 262,144 keys, in 256-row oracle blocks)
    sampled_parity(csa, "c5", heads=[(0, 0), (0, 3)], n_rows=16, tail=2048)
