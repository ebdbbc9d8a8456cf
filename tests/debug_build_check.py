"""Small cases of every entry point through the ATTN_DEBUG build of the
library, against the float64 oracle: the bounds checks must stay silent
(status ATTN_OK) and, since the debug build fills every output with NaN
before its kernels run, an element no kernel writes would fail the
comparison. Run by tests/test_gpu_debug.py in a child process with
CSA_ATTN_DEBUG=1 (the package loads one library per process)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import causal_softmax_attention_b200 as csa  # noqa: E402
import oracle  # noqa: E402
from seeded_inputs import as_f64, block_mask, draw, draw_rect  # noqa: E402

TOL = {"f32": 1e-5, "bf16": 2e-2}


def rel(a, b, scale=None):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    denom = np.abs(b).max() if scale is None else scale
    return float(np.abs(a - b).max() / max(denom, 1e-30))


def check(tag, got, ref, tol, scale=None):
    g = as_f64(got.cpu())
    assert np.isfinite(g).all(), f"{tag}: an element was not written (NaN fill visible)"
    e = rel(g, ref, scale)
    assert e <= tol, f"{tag}: rel err {e:.3e} > {tol}"


def square(dtype, B, H, N, d, causal, seed):
    q, k, v, do = draw(B, H, N, d, seed, dtype)
    dev = [t.cuda() for t in (q, k, v, do)]
    o, lse = csa.forward(*dev[:3], causal)
    ws = csa.new_workspace(dev[0])
    dq, dk, dv = (torch.empty_like(dev[0]) for _ in range(3))
    csa.attn_bwd(dev[0], dev[1], dev[2], o, dev[3], lse, dq, dk, dv, ws, causal)
    torch.cuda.synchronize()
    assert csa.attn_fwd_last_status() == 0 and csa.attn_last_status(ws) == 0, "status"
    ref = oracle.backward(*(as_f64(t) for t in (q, k, v, do)), d ** -0.5, causal)
    gs = max(np.abs(ref[n]).max() for n in ("dQ", "dK", "dV"))
    check(f"{dtype} {N} O", o, ref["O"], TOL[dtype])
    for name, t in (("dQ", dq), ("dK", dk), ("dV", dv)):
        check(f"{dtype} {N} {name}", t, ref[name], TOL[dtype], gs)


def rect():
    q, k, v, do = draw_rect(2, 1, 200, 700, 64, 31, "bf16")
    dev = [t.cuda() for t in (q, k, v, do)]
    o, lse = csa.forward_rect(*dev[:3], 333, True)
    dq, dk, dv = csa.backward_rect(dev[0], dev[1], dev[2], o, dev[3], lse, 333, True)
    torch.cuda.synchronize()
    assert csa.attn_fwd_last_status() == 0
    ref = oracle.backward(*(as_f64(t) for t in (q, k, v, do)), 0.125, True, q_offset=333)
    gs = max(np.abs(ref[n]).max() for n in ("dQ", "dK", "dV"))
    for name, t in (("dQ", dq), ("dK", dk), ("dV", dv)):
        check(f"rect {name}", t, ref[name], TOL["bf16"], gs)


def masked():
    B, H, N, d = 1, 2, 6 * 128 + 40, 64
    q, k, v, do = draw(B, H, N, d, 32, "bf16")
    bm = block_mask("window:3", N)
    dev = [t.cuda() for t in (q, k, v, do)]
    mask = torch.from_numpy(bm).cuda()
    o = torch.empty_like(dev[0])
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    csa.attn_fwd_masked(*dev[:3], o, lse, mask)
    g = [torch.empty_like(dev[0]) for _ in range(3)]
    ws = csa.new_workspace(dev[0])
    csa.attn_bwd_masked(dev[0], dev[1], dev[2], o, dev[3], lse, *g, mask, ws)
    torch.cuda.synchronize()
    assert csa.attn_fwd_last_status() == 0 and csa.attn_last_status(ws) == 0
    ref = oracle.backward(*(as_f64(t) for t in (q, k, v, do)), d ** -0.5,
                          keep=oracle.block_mask_keep(bm, N))
    gs = max(np.abs(ref[n]).max() for n in ("dQ", "dK", "dV"))
    for name, t in zip(("dQ", "dK", "dV"), g):
        check(f"masked {name}", t, ref[name], TOL["bf16"], gs)


def double_backward(dtype, N, d):
    q, k, v, do = draw(1, 1, N, d, 33, dtype)
    uq, uk, uv, _ = draw(1, 1, N, d, 34, dtype)
    dev = [t.cuda() for t in (q, k, v, do, uq, uk, uv)]
    o, lse = csa.forward(*dev[:3])
    outs = csa.backward_over_backward(dev[0], dev[1], dev[2], o, dev[3], lse, *dev[4:])
    torch.cuda.synchronize()
    ref = oracle.double_backward(*(as_f64(t) for t in (q, k, v, do, uq, uk, uv)), d ** -0.5)
    gs = max(np.abs(ref[n]).max() for n in ("gQ", "gK", "gV", "gdO"))
    for name, t in zip(("gQ", "gK", "gV", "gdO"), outs):
        check(f"bob {dtype} {name}", t, ref[name], TOL[dtype], gs)


def main():
    assert csa.DEBUG, "CSA_ATTN_DEBUG=1 must select the debug library"
    square("bf16", 2, 2, 333, 64, True, 21)
    square("bf16", 1, 3, 130, 128, False, 22)
    square("bf16", 1, 1, 257, 32, True, 23)
    square("f32", 1, 2, 201, 48, True, 24)
    rect()
    masked()
    double_backward("bf16", 300, 64)
    double_backward("f32", 90, 32)
    print("debug build ok")


if __name__ == "__main__":
    main()
