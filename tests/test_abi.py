"""CPU-side checks of the C ABI: the library loads, exports every function that
include/attn.h declares, sizes its workspace as documented and rejects bad
arguments before touching the GPU (every call below returns during argument
checking, so no CUDA call is made)."""
import ctypes
import math
import os
import re

import pytest

import causal_softmax_attention_b200 as csa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fname in os.listdir(os.path.join(ROOT, "include")):
        if not fname.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fname)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(attn_\w+)\s*\(", text):
            names.add(m.group(1))
    return names


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("attn_fwd", "attn_bwd", "attn_bwd_workspace_bytes", "attn_last_status",
                     "attn_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(csa.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(csa.EXPORTED) >= declared_functions()


def test_status_strings():
    assert csa.status_string(csa.ATTN_OK) == "ok"
    assert "timed out" in csa.status_string(csa.ATTN_ERR_TIMEOUT)
    assert csa.status_string(12345) == "unknown status"


def up(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("B,H,N,d", [(1, 1, 256, 64), (12, 4, 64, 32), (2, 16, 16384, 128),
                                     (1, 4, 262144, 64), (3, 5, 1000, 128), (1, 1, 1, 32)])
def test_workspace_bytes(B, H, N, d):
    Np = (N + 127) // 128 * 128
    rows = B * H * Np * 4
    f32 = 256 + up(rows) + up(rows)
    assert csa.attn_bwd_workspace_bytes(B, H, N, d, csa.ATTN_F32) == f32
    assert csa.attn_bwd_workspace_bytes(B, H, N, d, csa.ATTN_BF16) == f32 + up(rows * d)


def test_workspace_is_linear_in_n():
    a = csa.attn_bwd_workspace_bytes(1, 4, 131072, 64, csa.ATTN_BF16)
    b = csa.attn_bwd_workspace_bytes(1, 4, 262144, 64, csa.ATTN_BF16)
    assert abs(b / a - 2.0) < 1e-3


@pytest.mark.parametrize("args,status", [
    ((0, 1, 64, 64, 1), 0), ((1, 1, 0, 64, 1), 0), ((1, 1, 64, 48, 1), 0),
    ((1, 1, 64, 256, 0), 0), ((1, 1, 64, 64, 7), 0)])
def test_workspace_bytes_rejects(args, status):
    assert csa.attn_bwd_workspace_bytes(*args) == status


L = csa.library()
A = 1 << 20  # a 16-byte aligned stand-in address; never dereferenced (calls fail in checks)


def bwd(**over):
    a = dict(q=A, k=A, v=A, o=A, do=A, lse=A, dq=A, dk=A, dv=A, B=1, H=1, N=64, d=64,
             causal=1, scale=0.125, dt=csa.ATTN_BF16, ws=A, wsb=1 << 30, stream=None)
    a.update(over)
    return L.attn_bwd(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"],
                      a["dv"], a["B"], a["H"], a["N"], a["d"], a["causal"], a["scale"], a["dt"],
                      a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("over,status", [
    (dict(q=None), csa.ATTN_ERR_INVALID),
    (dict(dv=None), csa.ATTN_ERR_INVALID),
    (dict(k=A + 8), csa.ATTN_ERR_INVALID),
    (dict(B=0), csa.ATTN_ERR_INVALID),
    (dict(H=-1), csa.ATTN_ERR_INVALID),
    (dict(N=0), csa.ATTN_ERR_INVALID),
    (dict(scale=math.nan), csa.ATTN_ERR_INVALID),
    (dict(scale=math.inf), csa.ATTN_ERR_INVALID),
    (dict(d=48), csa.ATTN_ERR_UNSUPPORTED),
    (dict(d=256, dt=csa.ATTN_F32), csa.ATTN_ERR_UNSUPPORTED),
    (dict(dt=3), csa.ATTN_ERR_UNSUPPORTED),
    (dict(ws=None), csa.ATTN_ERR_INVALID),
    (dict(wsb=100), csa.ATTN_ERR_INVALID),
])
def test_bwd_rejects_bad_arguments(over, status):
    assert bwd(**over) == status


def test_fwd_rejects_bad_arguments():
    f = L.attn_fwd
    assert f(None, A, A, A, A, 1, 1, 64, 64, 1, 0.125, 1, None) == csa.ATTN_ERR_INVALID
    assert f(A, A, A, A, A + 4, 1, 1, 64, 64, 1, 0.125, 1, None) == csa.ATTN_ERR_INVALID
    assert f(A, A, A, A, A, 1, 1, 64, 96, 1, 0.125, 1, None) == csa.ATTN_ERR_UNSUPPORTED
    assert f(A, A, A, A, A, 1, 1, 64, 64, 1, math.nan, 1, None) == csa.ATTN_ERR_INVALID


def test_stage_entry_points_reject_bad_arguments():
    assert L.attn_bwd_preprocess(A, None, A, 1, 1, 64, 64, 1, A, 1 << 30, None) == csa.ATTN_ERR_INVALID
    assert L.attn_bwd_main(A, A, A, A, A, A, A, 1, 1, 64, 64, 1, 0.1, 1, A, 10, None) == csa.ATTN_ERR_INVALID
    assert L.attn_bwd_dq_convert(A, 1, 1, 64, 40, 0.1, 1, A, 1 << 30, None) == csa.ATTN_ERR_UNSUPPORTED
    assert L.attn_last_status(None) == csa.ATTN_ERR_INVALID
    assert L.attn_test_arm_timeout(0) == csa.ATTN_ERR_INVALID


def test_masked_entry_points_reject_bad_arguments():
    # every call returns during argument checking (no CUDA call)
    f, b = L.attn_fwd_masked, L.attn_bwd_masked
    assert f(A, A, A, A, A, 1, 1, 300, 64, None, 0.125, 1, None) == csa.ATTN_ERR_INVALID
    assert f(A, A, A, A, A, 1, 1, 300, 64, A, 0.125, 0, None) == csa.ATTN_ERR_UNSUPPORTED
    assert f(A, A, A, A, A + 4, 1, 1, 300, 64, A, 0.125, 1, None) == csa.ATTN_ERR_INVALID
    assert f(A, A, A, A, A, 1, 1, 300, 96, A, 0.125, 1, None) == csa.ATTN_ERR_UNSUPPORTED
    args = [A] * 9 + [1, 1, 300, 64]
    assert b(*args, None, 0.125, 1, A, 1 << 30, None) == csa.ATTN_ERR_INVALID
    assert b(*args, A, 0.125, 0, A, 1 << 30, None) == csa.ATTN_ERR_UNSUPPORTED
    assert b(*args, A, math.nan, 1, A, 1 << 30, None) == csa.ATTN_ERR_INVALID
    assert b(*args, A, 0.125, 1, A, 16, None) == csa.ATTN_ERR_INVALID
    m = L.attn_bwd_main_masked
    args = [A] * 7 + [1, 1, 300, 64]
    assert m(*args, None, 0.125, 1, A, 1 << 30, None) == csa.ATTN_ERR_INVALID
    assert m(*args, A, 0.125, 0, A, 1 << 30, None) == csa.ATTN_ERR_UNSUPPORTED
    assert m(*args, A, math.nan, 1, A, 1 << 30, None) == csa.ATTN_ERR_INVALID
    assert m(*args, A, 0.125, 1, A, 16, None) == csa.ATTN_ERR_INVALID
    assert m(*([A] * 6 + [A + 8, 1, 1, 300, 64]), A, 0.125, 1, A, 1 << 30, None) == csa.ATTN_ERR_INVALID


def test_strided_entry_points_reject_bad_strides():
    # every call returns during argument checking (no CUDA call)
    f, b = L.attn_fwd_strided, L.attn_bwd_strided
    good = (ctypes.c_longlong * 3)(300 * 64 * 2, 64, 2 * 64)
    bad = {
        "null": None,
        "zero": (ctypes.c_longlong * 3)(0, 64, 128),
        "negative": (ctypes.c_longlong * 3)(300 * 128, -64, 128),
        "row closer than d": (ctypes.c_longlong * 3)(300 * 64, 64, 32),
        "bf16 not 16-byte": (ctypes.c_longlong * 3)(300 * 128, 68, 128),
        "beyond the map limit": (ctypes.c_longlong * 3)(1 << 36, 64, 128),
    }
    fargs = [A] * 5 + [1, 2, 300, 64]
    bargs = [A] * 9 + [1, 2, 300, 64]
    for name, st in bad.items():
        p = ctypes.addressof(st) if st is not None else None
        g = ctypes.addressof(good)
        assert f(*fargs, p, g, 1, 0.125, 1, None) == csa.ATTN_ERR_INVALID, name
        assert f(*fargs, g, p, 1, 0.125, 1, None) == csa.ATTN_ERR_INVALID, name
        assert b(*bargs, p, g, 1, 0.125, 1, A, 1 << 30, None) == csa.ATTN_ERR_INVALID, name
        assert b(*bargs, g, p, 1, 0.125, 1, A, 1 << 30, None) == csa.ATTN_ERR_INVALID, name
    # shape checks come first; an unsupported head size stays unsupported
    g = ctypes.addressof(good)
    assert f(*([A] * 5 + [1, 2, 300, 96]), g, g, 1, 0.125, 1, None) == csa.ATTN_ERR_UNSUPPORTED


def test_row_strides_of_views():
    import torch
    x = torch.empty(2, 5, 3, 64)  # [B, N, H, d]
    assert csa.row_strides(x.permute(0, 2, 1, 3)) == (5 * 3 * 64, 64, 3 * 64)
    qkv = torch.empty(2, 5, 3, 4, 32)  # packed [B, N, 3, H, d]
    assert csa.row_strides(qkv[:, :, 1].permute(0, 2, 1, 3)) == (5 * 3 * 4 * 32, 32, 3 * 4 * 32)
    with pytest.raises(ValueError):
        csa.row_strides(x.permute(0, 3, 1, 2))


def test_double_backward_entry_point_rejects_bad_arguments():
    # every call returns during argument checking (no CUDA call)
    f = L.attn_bwd_bwd
    need = L.attn_bwd_bwd_workspace_bytes(1, 2, 300, 64, 0)
    assert need >= 2 * 2 * 384 * 4
    # bf16 (tensor-core kernels) takes the same workspace: no dQ accumulator
    assert L.attn_bwd_bwd_workspace_bytes(1, 2, 300, 64, 1) == need
    assert L.attn_bwd_bwd_workspace_bytes(1, 2, 300, 48, 1) == 0  # bf16 d outside {32, 64, 128}
    ptrs = [A] * 13
    assert f(*ptrs, 1, 2, 300, 48, 1, 0.125, 1, A, 1 << 30, None) == csa.ATTN_ERR_UNSUPPORTED
    assert f(*([A] * 9 + [A + 4] + [A] * 3), 1, 2, 300, 64, 1, 0.125, 1, A, 1 << 30,
             None) == csa.ATTN_ERR_INVALID  # bf16 tensors must be 16-byte aligned
    assert f(*ptrs, 1, 2, 300, 64, 1, 0.125, 1, A, need - 1, None) == csa.ATTN_ERR_INVALID
    assert f(*ptrs, 1, 2, 300, 64, 1, 0.125, 0, A, need - 1, None) == csa.ATTN_ERR_INVALID
    assert f(*ptrs, 1, 2, 300, 64, 1, math.inf, 0, A, need, None) == csa.ATTN_ERR_INVALID
    assert f(*ptrs, 1, 2, 300, 200, 1, 0.125, 0, A, need, None) == csa.ATTN_ERR_UNSUPPORTED
    assert f(*([A] * 12 + [None]), 1, 2, 300, 64, 1, 0.125, 0, A, need, None) == csa.ATTN_ERR_INVALID
    assert f(*([A] * 5 + [A + 4] + [A] * 7), 1, 2, 300, 64, 1, 0.125, 0, A, need,
             None) == csa.ATTN_ERR_INVALID  # lse must be 16-byte aligned
    assert f(*ptrs, 1, 2, 300, 64, 1, 0.125, 0, A + 8, need, None) == csa.ATTN_ERR_INVALID


def test_rectangular_entry_points_reject_bad_arguments():
    # every call returns during argument checking (no CUDA call)
    f, b = L.attn_fwd_rect, L.attn_bwd_rect
    ws = 1 << 30
    assert f(A, A, A, A, A, 1, 1, 0, 64, 64, 0, 1, 0.125, 1, None) == csa.ATTN_ERR_INVALID
    assert f(A, A, A, A, A, 1, 1, 64, 0, 64, 0, 1, 0.125, 1, None) == csa.ATTN_ERR_INVALID
    assert f(A, A, A, A, A, 1, 1, 64, 64, 64, -1, 1, 0.125, 1, None) == csa.ATTN_ERR_INVALID
    assert f(A, A, A, A, A, 1, 1, 64, 64, 64, (1 << 30) + 1, 1, 0.125, 1, None) == csa.ATTN_ERR_INVALID
    assert f(None, A, A, A, A, 1, 1, 64, 200, 64, 0, 1, 0.125, 1, None) == csa.ATTN_ERR_INVALID
    assert f(A, A, A, A, A, 1, 1, 64, 200, 96, 0, 1, 0.125, 1, None) == csa.ATTN_ERR_UNSUPPORTED
    assert b(A, A, A, A, A, A, A, A, A, 1, 1, 64, 200, 64, -3, 1, 0.125, 1, A, ws, None) == csa.ATTN_ERR_INVALID
    assert b(A, A, A, A, A, A, A, A, A, 1, 1, 64, 0, 64, 0, 1, 0.125, 1, A, ws, None) == csa.ATTN_ERR_INVALID
    # the workspace is sized by the query rows: one sized for fewer rows is refused
    small = csa.attn_bwd_workspace_bytes(1, 1, 64, 64, csa.ATTN_BF16)
    assert b(A, A, A, A, A, A, A, A, A, 1, 1, 300, 64, 64, 0, 1, 0.125, 1, A, small, None) == csa.ATTN_ERR_INVALID
    assert b(A, A, A, A, A, A, A, A, A, 1, 1, 64, 64, 64, 0, 1, math.nan, 1, A, ws, None) == csa.ATTN_ERR_INVALID


def test_debug_build_exports_the_same_boundary():
    # the ATTN_DEBUG variant (built beside the release library) exports every
    # declared symbol, names the bounds status, and checks arguments the same
    # way before any CUDA call
    from causal_softmax_attention_b200.build import DEBUG_LIB_PATH
    dbg = ctypes.CDLL(DEBUG_LIB_PATH)
    for name in declared_functions():
        assert hasattr(dbg, name), name
    dbg.attn_status_string.restype = ctypes.c_char_p
    assert b"bounds" in dbg.attn_status_string(csa.ATTN_ERR_BOUNDS)
    assert b"bounds" in L.attn_status_string(csa.ATTN_ERR_BOUNDS)
    f = dbg.attn_fwd
    f.argtypes = L.attn_fwd.argtypes
    assert f(None, A, A, A, A, 1, 1, 64, 64, 1, 0.125, 1, None) == csa.ATTN_ERR_INVALID
    assert f(A, A, A, A, A, 1, 1, 64, 96, 1, 0.125, 1, None) == csa.ATTN_ERR_UNSUPPORTED
