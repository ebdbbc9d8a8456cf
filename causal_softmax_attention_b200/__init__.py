"""Python binding of the B200 causal softmax attention library (libcsa_attn.so).

The functions here marshal arguments for the C ABI in include/attn.h and do
nothing else: every step of the forward and backward runs in the library's
CUDA kernels. Tensor arguments are torch tensors (device memory and streams
are torch's plumbing); raw-pointer variants take integers. If the shared
library is missing, importing this package raises: there is no CPU fallback.

Build the library with ``python causal_softmax_attention_b200/build.py``.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .build import LIB_PATH

ATTN_OK = 0
ATTN_ERR_INVALID = -1
ATTN_ERR_UNSUPPORTED = -2
ATTN_ERR_CUDA = -3
ATTN_ERR_TIMEOUT = -4
ATTN_F32 = 0
ATTN_BF16 = 1

_DTYPES = {torch.float32: ATTN_F32, torch.bfloat16: ATTN_BF16}


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python causal_softmax_attention_b200/build.py` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "attn_fwd": (i, [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]),
        "attn_bwd_workspace_bytes": (sz, [i, i, i, i, i]),
        "attn_bwd": (i, [vp] * 9 + [i, i, i, i, i, f, i, vp, sz, vp]),
        "attn_bwd_preprocess": (i, [vp, vp, vp, i, i, i, i, i, vp, sz, vp]),
        "attn_bwd_main": (i, [vp] * 7 + [i, i, i, i, i, f, i, vp, sz, vp]),
        "attn_bwd_dq_convert": (i, [vp, i, i, i, i, f, i, vp, sz, vp]),
        "attn_last_status": (i, [vp]),
        "attn_fwd_last_status": (i, []),
        "attn_status_string": (ctypes.c_char_p, [i]),
        "attn_test_arm_timeout": (i, [ctypes.c_ulonglong]),
        "attn_bwd_noalloc": (i, [vp] * 9 + [i, i, i, i, i, f, i, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
EXPORTED = ("attn_fwd", "attn_bwd_workspace_bytes", "attn_bwd", "attn_bwd_preprocess",
            "attn_bwd_main", "attn_bwd_dq_convert", "attn_last_status", "attn_fwd_last_status",
            "attn_status_string", "attn_test_arm_timeout", "attn_bwd_noalloc")


def library() -> ctypes.CDLL:
    return _lib


def status_string(status: int) -> str:
    return _lib.attn_status_string(int(status)).decode()


def _ptr(t) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _shape(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(int(x) for x in q.shape)


def _check(status: int, where: str) -> None:
    if status != ATTN_OK:
        raise AttnError(status, where)


def attn_bwd_workspace_bytes(B: int, H: int, N: int, d: int, dtype) -> int:
    dt = _DTYPES[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    return int(_lib.attn_bwd_workspace_bytes(B, H, N, d, dt))


def attn_fwd(q, k, v, o, lse, causal: bool = True, scale: float | None = None, stream=None,
             check: bool = True) -> int:
    """O, LSE <- forward of q, k, v ([B, H, N, d] contiguous CUDA tensors, f32 or bf16)."""
    B, H, N, d = _shape(q)
    scale = d ** -0.5 if scale is None else scale
    st = _lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, int(causal),
                       float(scale), _DTYPES[q.dtype], _stream(stream))
    if check:
        _check(st, "attn_fwd")
    return st


def attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, causal: bool = True,
             scale: float | None = None, stream=None, check: bool = True) -> int:
    """dQ, dK, dV <- backward; `workspace` is a CUDA uint8 tensor of
    attn_bwd_workspace_bytes bytes."""
    B, H, N, d = _shape(q)
    scale = d ** -0.5 if scale is None else scale
    st = _lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                       _ptr(dk), _ptr(dv), B, H, N, d, int(causal), float(scale),
                       _DTYPES[q.dtype], _ptr(workspace), int(workspace.numel()),
                       _stream(stream))
    if check:
        _check(st, "attn_bwd")
    return st


def attn_bwd_preprocess(o, dout, lse, workspace, stream=None) -> int:
    B, H, N, d = _shape(o)
    st = _lib.attn_bwd_preprocess(_ptr(o), _ptr(dout), _ptr(lse), B, H, N, d, _DTYPES[o.dtype],
                                  _ptr(workspace), int(workspace.numel()), _stream(stream))
    _check(st, "attn_bwd_preprocess")
    return st


def attn_bwd_main(q, k, v, dout, dq, dk, dv, workspace, causal: bool = True,
                  scale: float | None = None, stream=None) -> int:
    B, H, N, d = _shape(q)
    scale = d ** -0.5 if scale is None else scale
    st = _lib.attn_bwd_main(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                            B, H, N, d, int(causal), float(scale), _DTYPES[q.dtype],
                            _ptr(workspace), int(workspace.numel()), _stream(stream))
    _check(st, "attn_bwd_main")
    return st


def attn_bwd_dq_convert(dq, workspace, scale: float | None = None, stream=None) -> int:
    B, H, N, d = _shape(dq)
    scale = d ** -0.5 if scale is None else scale
    st = _lib.attn_bwd_dq_convert(_ptr(dq), B, H, N, d, float(scale), _DTYPES[dq.dtype],
                                  _ptr(workspace), int(workspace.numel()), _stream(stream))
    _check(st, "attn_bwd_dq_convert")
    return st


def attn_last_status(workspace) -> int:
    return int(_lib.attn_last_status(_ptr(workspace)))


def attn_fwd_last_status() -> int:
    return int(_lib.attn_fwd_last_status())


def attn_test_arm_timeout(wait_limit_ns: int) -> int:
    return int(_lib.attn_test_arm_timeout(int(wait_limit_ns)))


def new_workspace(q: torch.Tensor) -> torch.Tensor:
    """Allocate (through torch) a workspace for attn_bwd on q's shape and device."""
    B, H, N, d = _shape(q)
    nbytes = attn_bwd_workspace_bytes(B, H, N, d, q.dtype)
    if nbytes == 0:
        raise AttnError(ATTN_ERR_INVALID, "attn_bwd_workspace_bytes")
    return torch.empty(nbytes, dtype=torch.uint8, device=q.device)


def forward(q, k, v, causal: bool = True, scale: float | None = None):
    """Convenience: allocate O and LSE with torch and run attn_fwd."""
    B, H, N, d = _shape(q)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=q.device)
    attn_fwd(q, k, v, o, lse, causal, scale)
    return o, lse


def backward(q, k, v, o, dout, lse, causal: bool = True, scale: float | None = None,
             workspace=None):
    """Convenience: allocate dQ, dK, dV (and a workspace) and run attn_bwd."""
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = new_workspace(q) if workspace is None else workspace
    attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, ws, causal, scale)
    return dq, dk, dv
