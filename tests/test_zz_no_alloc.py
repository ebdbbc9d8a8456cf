"""attn_bwd_noalloc, the backward for callers that cannot allocate device memory
(for example a plugin inside a framework that owns all device memory through
its own pool, or latency-critical code that cannot pay for cudaMalloc). It
takes its scratch from a fixed array inside the library instead of a caller
workspace; its results must match attn_bwd's, call after call, whatever shape
the previous call left its row terms and accumulator in.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes on its own.
"""
import numpy as np
import pytest
import torch

from seeded_inputs import as_f64, draw

pytestmark = pytest.mark.gpu


def _rel(a, b):
    a, b = as_f64(a.cpu()), as_f64(b.cpu())
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import causal_softmax_attention_b200 as csa
    return csa, csa.library()


def _noalloc(csa, lib, q, k, v, o, do, lse, outs, scale):
    B, H, N, d = q.shape
    dt = csa.ATTN_BF16 if q.dtype == torch.bfloat16 else csa.ATTN_F32
    return lib.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                do.data_ptr(), lse.data_ptr(), outs[0].data_ptr(),
                                outs[1].data_ptr(), outs[2].data_ptr(), B, H, N, d, 1, scale, dt,
                                torch.cuda.current_stream().cuda_stream)


def _check_against_attn_bwd(csa, lib, B, H, N, d, dtype, seed, tol, calls=1):
    scale = d ** -0.5
    q, k, v, do = (t.cuda() for t in draw(B, H, N, d, seed, dtype))
    o, lse = csa.forward(q, k, v, True, scale)
    want = csa.backward(q, k, v, o, do, lse, True, scale)  # attn_bwd with a workspace
    for _ in range(calls):  # the shared scratch keeps the previous call's contents
        got = [torch.full_like(q, float("nan")) for _ in range(3)]
        st = _noalloc(csa, lib, q, k, v, o, do, lse, got, scale)
        assert st == csa.ATTN_OK, csa.status_string(st)
        torch.cuda.synchronize()
        assert lib.attn_bwd_noalloc_last_status() == csa.ATTN_OK
        for g, w in zip(got, want):
            assert _rel(g, w) <= tol


@pytest.mark.parametrize("dtype,tol", [("bf16", 2e-2), ("f32", 1e-5)])
def test_no_alloc_matches_attn_bwd_twice(dtype, tol):
    csa, lib = _lib()
    _check_against_attn_bwd(csa, lib, 2, 3, 700, 64, dtype, 77, tol, calls=2)


def test_no_alloc_across_shapes_and_at_its_limit():
    # calls of different shapes place the row terms and the dQ accumulator at
    # different offsets of the array: a larger call, then smaller ones, then
    # the largest bf16 shape of one head at d = 128 that fits (its workspace
    # is just under the array's size), then a small one again
    csa, lib = _lib()
    limit = 16 << 20  # ATTN_BWD_NOALLOC_SCRATCH_BYTES
    n_max = 32256
    assert csa.attn_bwd_workspace_bytes(1, 1, n_max, 128, torch.bfloat16) <= limit
    assert csa.attn_bwd_workspace_bytes(1, 1, n_max + 1, 128, torch.bfloat16) > limit
    for (B, H, N, d, seed) in ((1, 6, 3000, 128, 81), (2, 1, 257, 32, 82), (1, 2, 900, 64, 83),
                               (1, 1, n_max, 128, 84), (3, 1, 129, 64, 85)):
        _check_against_attn_bwd(csa, lib, B, H, N, d, "bf16", seed, 2e-2)


def test_no_alloc_rejects_shapes_beyond_its_scratch():
    csa, lib = _lib()
    x = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = x.data_ptr()
    # 1 x 32 heads x 16,384 tokens x d=128 needs far more than 16 MiB; one
    # head of 32,257 tokens at d = 128 needs just over it
    for (H, N) in ((32, 16384), (1, 32257)):
        st = lib.attn_bwd_noalloc(p, p, p, p, p, p, p, p, p, 1, H, N, 128, 1, 0.08,
                                  csa.ATTN_BF16, None)
        assert st == csa.ATTN_ERR_INVALID


def test_no_alloc_reports_a_device_timeout():
    # a timed-out call (armed through the test hook: bounded waits that run
    # out, no fault) shows in the status word; the next call is clean
    csa, lib = _lib()
    B, H, N, d = 1, 1, 256, 64
    q, k, v, do = (t.cuda() for t in draw(B, H, N, d, 86, "bf16"))
    o, lse = csa.forward(q, k, v)
    got = [torch.empty_like(q) for _ in range(3)]
    assert csa.attn_test_arm_timeout(50_000_000) == csa.ATTN_OK  # ~25 ms of SM cycles
    assert _noalloc(csa, lib, q, k, v, o, do, lse, got, d ** -0.5) == csa.ATTN_OK
    assert lib.attn_bwd_noalloc_last_status() == csa.ATTN_ERR_TIMEOUT
    assert _noalloc(csa, lib, q, k, v, o, do, lse, got, d ** -0.5) == csa.ATTN_OK
    assert lib.attn_bwd_noalloc_last_status() == csa.ATTN_OK
