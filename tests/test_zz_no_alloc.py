"""attn_bwd_noalloc, the backward for callers that cannot allocate device memory
(for example a plugin inside a framework that owns all device memory through
its own pool, or latency-critical code that cannot pay for cudaMalloc). It
takes its scratch from a fixed array inside the library instead of a caller
workspace; its results must match attn_bwd's, call after call.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

from seeded_inputs import as_f64, draw

pytestmark = pytest.mark.gpu


def _rel(a, b):
    a, b = as_f64(a.cpu()), as_f64(b.cpu())
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


@pytest.mark.parametrize("dtype,tol", [("bf16", 2e-2), ("f32", 1e-5)])
def test_no_alloc_matches_attn_bwd_twice(dtype, tol):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import causal_softmax_attention_b200 as csa

    lib = csa.library()
    B, H, N, d = 2, 3, 700, 64
    scale = d ** -0.5
    q, k, v, do = (t.cuda() for t in draw(B, H, N, d, 77, dtype))
    o, lse = csa.forward(q, k, v, True, scale)
    want = csa.backward(q, k, v, o, do, lse, True, scale)  # attn_bwd with a workspace
    dt = csa.ATTN_BF16 if dtype == "bf16" else csa.ATTN_F32
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):  # the shared scratch keeps the previous call's contents
        got = [torch.full_like(q, float("nan")) for _ in range(3)]
        st = lib.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  do.data_ptr(), lse.data_ptr(), got[0].data_ptr(),
                                  got[1].data_ptr(), got[2].data_ptr(), B, H, N, d, 1, scale,
                                  dt, stream)
        assert st == csa.ATTN_OK, csa.status_string(st)
        torch.cuda.synchronize()
        for g, w in zip(got, want):
            assert _rel(g, w) <= tol


def test_no_alloc_rejects_shapes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import causal_softmax_attention_b200 as csa

    lib = csa.library()
    x = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = x.data_ptr()
    # 1 x 32 heads x 16,384 tokens x d=128 needs far more than 16 MiB
    st = lib.attn_bwd_noalloc(p, p, p, p, p, p, p, p, p, 1, 32, 16384, 128, 1, 0.08,
                              csa.ATTN_BF16, None)
    assert st == csa.ATTN_ERR_INVALID
