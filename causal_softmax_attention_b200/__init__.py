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

from .build import DEBUG_LIB_PATH, LIB_PATH

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


# CSA_ATTN_DEBUG=1 loads the ATTN_DEBUG build (device-side bounds checks
# reporting ATTN_ERR_BOUNDS, outputs filled with NaN before each call).
DEBUG = os.environ.get("CSA_ATTN_DEBUG") == "1"
ATTN_ERR_BOUNDS = -5


def _load() -> ctypes.CDLL:
    path = DEBUG_LIB_PATH if DEBUG else LIB_PATH
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python causal_softmax_attention_b200/build.py"
            f"{' --debug' if DEBUG else ''}` (there is no CPU fallback)")
    lib = ctypes.CDLL(path)
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
        "attn_test_exp2": (i, [vp, vp, vp, i, vp]),
        "attn_bwd_noalloc": (i, [vp] * 9 + [i, i, i, i, i, f, i, vp]),
        "attn_bwd_noalloc_last_status": (i, []),
        "attn_fwd_masked": (i, [vp] * 5 + [i, i, i, i, vp, f, i, vp]),
        "attn_bwd_masked": (i, [vp] * 9 + [i, i, i, i, vp, f, i, vp, sz, vp]),
        "attn_bwd_main_masked": (i, [vp] * 7 + [i, i, i, i, vp, f, i, vp, sz, vp]),
        "attn_fwd_strided": (i, [vp] * 5 + [i, i, i, i, vp, vp, i, f, i, vp]),
        "attn_bwd_strided": (i, [vp] * 9 + [i, i, i, i, vp, vp, i, f, i, vp, sz, vp]),
        "attn_fwd_rect": (i, [vp] * 5 + [i] * 7 + [f, i, vp]),
        "attn_bwd_rect": (i, [vp] * 9 + [i] * 7 + [f, i, vp, sz, vp]),
        "attn_bwd_bwd_workspace_bytes": (sz, [i, i, i, i, i]),
        "attn_bwd_bwd": (i, [vp] * 13 + [i, i, i, i, i, f, i, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
EXPORTED = ("attn_fwd", "attn_bwd_workspace_bytes", "attn_bwd", "attn_bwd_preprocess",
            "attn_bwd_main", "attn_bwd_dq_convert", "attn_last_status", "attn_fwd_last_status",
            "attn_status_string", "attn_test_arm_timeout", "attn_bwd_noalloc",
            "attn_bwd_noalloc_last_status", "attn_fwd_masked",
            "attn_bwd_masked", "attn_bwd_main_masked", "attn_fwd_strided", "attn_bwd_strided",
            "attn_bwd_bwd_workspace_bytes", "attn_bwd_bwd", "attn_fwd_rect", "attn_bwd_rect",
            "attn_test_exp2")


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


def attn_bwd_main_masked(q, k, v, dout, dq, dk, dv, block_mask, workspace,
                         scale: float | None = None, stream=None) -> int:
    """The main stage of attn_bwd_masked (between attn_bwd_preprocess and
    attn_bwd_dq_convert); `block_mask` as in attn_fwd_masked."""
    B, H, N, d = _shape(q)
    scale = d ** -0.5 if scale is None else scale
    st = _lib.attn_bwd_main_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk),
                                   _ptr(dv), B, H, N, d, _ptr(block_mask), float(scale),
                                   _DTYPES[q.dtype], _ptr(workspace), int(workspace.numel()),
                                   _stream(stream))
    _check(st, "attn_bwd_main_masked")
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


def attn_test_arm_timeout(wait_limit_cycles: int) -> int:
    """Arm the one-shot timeout of the next bf16 backward; each of its device
    waits is bounded by `wait_limit_cycles` SM clock cycles."""
    return int(_lib.attn_test_arm_timeout(int(wait_limit_cycles)))


def new_workspace(q: torch.Tensor) -> torch.Tensor:
    """Allocate (through torch) a workspace for attn_bwd on q's shape and device."""
    B, H, N, d = _shape(q)
    nbytes = attn_bwd_workspace_bytes(B, H, N, d, q.dtype)
    if nbytes == 0:
        raise AttnError(ATTN_ERR_INVALID, "attn_bwd_workspace_bytes")
    return torch.empty(nbytes, dtype=torch.uint8, device=q.device)


def row_strides(t: torch.Tensor) -> tuple:
    """Element strides (b, h, n) of a [B, H, N, d] view whose channels are
    contiguous, e.g. x.permute(0, 2, 1, 3) of a [B, N, H, d] tensor."""
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("expected a [B, H, N, d] view with unit channel stride")
    return tuple(int(x) for x in t.stride()[:3])


def _strides_arg(tensors, what: str):
    st = {row_strides(t) for t in tensors}
    if len(st) != 1:
        raise ValueError(f"{what} must share one stride set, got {sorted(st)}")
    return (ctypes.c_longlong * 3)(*st.pop())


def attn_fwd_strided(q, k, v, o, lse, causal: bool = True, scale: float | None = None,
                     stream=None, check: bool = True) -> int:
    """attn_fwd on [B, H, N, d] views of any row strides: q, k, v share one
    stride set (e.g. slices of a packed projection), o may have its own."""
    B, H, N, d = _shape(q)
    scale = d ** -0.5 if scale is None else scale
    qs, os_ = _strides_arg((q, k, v), "q, k, v"), _strides_arg((o,), "o")
    st = _lib.attn_fwd_strided(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                               ctypes.addressof(qs), ctypes.addressof(os_), int(causal),
                               float(scale), _DTYPES[q.dtype], _stream(stream))
    if check:
        _check(st, "attn_fwd_strided")
    return st


def attn_bwd_strided(q, k, v, o, dout, lse, dq, dk, dv, workspace, causal: bool = True,
                     scale: float | None = None, stream=None, check: bool = True) -> int:
    """attn_bwd on strided views: q, k, v, dq, dk, dv share one stride set,
    o and dout another."""
    B, H, N, d = _shape(q)
    scale = d ** -0.5 if scale is None else scale
    qs = _strides_arg((q, k, v, dq, dk, dv), "q, k, v, dq, dk, dv")
    os_ = _strides_arg((o, dout), "o, dout")
    st = _lib.attn_bwd_strided(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                               _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, ctypes.addressof(qs),
                               ctypes.addressof(os_), int(causal), float(scale),
                               _DTYPES[q.dtype], _ptr(workspace), int(workspace.numel()),
                               _stream(stream))
    if check:
        _check(st, "attn_bwd_strided")
    return st


def attn_fwd_rect(q, k, v, o, lse, q_offset: int = 0, causal: bool = True,
                  scale: float | None = None, stream=None, check: bool = True) -> int:
    """O, LSE <- forward of N_q query rows ([B, H, N_q, d] q, o) over N_k keys
    ([B, H, N_k, d] k, v); query row r is position q_offset + r."""
    B, H, nq, d = _shape(q)
    nk = int(k.shape[2])
    scale = d ** -0.5 if scale is None else scale
    st = _lib.attn_fwd_rect(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, nq, nk, d,
                            int(q_offset), int(causal), float(scale), _DTYPES[q.dtype],
                            _stream(stream))
    if check:
        _check(st, "attn_fwd_rect")
    return st


def attn_bwd_rect(q, k, v, o, dout, lse, dq, dk, dv, workspace, q_offset: int = 0,
                  causal: bool = True, scale: float | None = None, stream=None,
                  check: bool = True) -> int:
    """dQ, dK, dV of attn_fwd_rect; `workspace` sized by
    attn_bwd_workspace_bytes(B, H, N_q, d, dtype)."""
    B, H, nq, d = _shape(q)
    nk = int(k.shape[2])
    scale = d ** -0.5 if scale is None else scale
    st = _lib.attn_bwd_rect(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                            _ptr(dk), _ptr(dv), B, H, nq, nk, d, int(q_offset), int(causal),
                            float(scale), _DTYPES[q.dtype], _ptr(workspace),
                            int(workspace.numel()), _stream(stream))
    if check:
        _check(st, "attn_bwd_rect")
    return st


def forward_rect(q, k, v, q_offset: int = 0, causal: bool = True, scale: float | None = None):
    """Convenience: allocate O and LSE and run attn_fwd_rect."""
    B, H, nq, d = _shape(q)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, nq, dtype=torch.float32, device=q.device)
    attn_fwd_rect(q, k, v, o, lse, q_offset, causal, scale)
    return o, lse


def backward_rect(q, k, v, o, dout, lse, q_offset: int = 0, causal: bool = True,
                  scale: float | None = None):
    """Convenience: allocate dQ, dK, dV and a workspace and run attn_bwd_rect."""
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    attn_bwd_rect(q, k, v, o, dout, lse, dq, dk, dv, new_workspace(q), q_offset, causal, scale)
    return dq, dk, dv


def attn_bwd_bwd(q, k, v, o, dout, lse, uq, uk, uv, gq, gk, gv, gdout, workspace,
                 causal: bool = True, scale: float | None = None, stream=None,
                 check: bool = True) -> int:
    """Backward-over-backward: gq, gk, gv, gdout <- the gradients of
    <uq, dQ> + <uk, dK> + <uv, dV> w.r.t. q, k, v, dout (f32)."""
    B, H, N, d = _shape(q)
    scale = d ** -0.5 if scale is None else scale
    st = _lib.attn_bwd_bwd(*(_ptr(t) for t in (q, k, v, o, dout, lse, uq, uk, uv, gq, gk, gv,
                                               gdout)),
                           B, H, N, d, int(causal), float(scale), _DTYPES[q.dtype],
                           _ptr(workspace), int(workspace.numel()), _stream(stream))
    if check:
        _check(st, "attn_bwd_bwd")
    return st


def backward_over_backward(q, k, v, o, dout, lse, uq, uk, uv, causal: bool = True,
                           scale: float | None = None):
    """Convenience: allocate the outputs and a workspace, run attn_bwd_bwd."""
    B, H, N, d = _shape(q)
    out = [torch.empty_like(q) for _ in range(4)]
    ws = torch.empty(max(1, int(_lib.attn_bwd_bwd_workspace_bytes(B, H, N, d,
                                                                  _DTYPES[q.dtype]))),
                     dtype=torch.uint8, device=q.device)
    attn_bwd_bwd(q, k, v, o, dout, lse, uq, uk, uv, *out, ws, causal, scale)
    return tuple(out)


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


def backward_host(hq, hk, hv, ho, hdout, hlse, hdq, hdk, hdv, dev, causal: bool = True,
                  scale: float | None = None, chunks: int = 8, stream=None, block_mask=None,
                  recompute_forward: bool = False):
    """dQ, dK, dV of inputs held in (pinned) HOST memory, results written to
    host tensors, through attn_bwd with the transfers overlapped.

    The (batch, head) pairs are split into up to `chunks` consecutive groups.
    Group c is copied to the device on one stream, its backward runs on a
    second once its inputs have landed, and its gradients are copied back on
    a third, so that the host->device copy of group c+1, the backward of
    group c and the device->host copy of group c-1 proceed together.

    `dev` is a dict of device buffers of the full shapes: q, k, v, o, dout
    ([B, H, N, d]), lse ([B, H, N]), dq, dk, dv, and `workspace` sized by
    attn_bwd_workspace_bytes for one group (chunk_workspace_bytes). The work
    starts after everything already queued on `stream` (default: the current
    stream) and `stream` waits for all of it to finish, so events recorded
    on `stream` around the call time the whole transfer and compute. With a
    `block_mask` (a device uint8 [T, T] tensor, as in attn_bwd_masked) each
    group runs attn_bwd_masked instead and `causal` is ignored. With
    `recompute_forward` the host O and LSE are not used (ho, hlse may be
    None): each group's forward runs on the device before its backward, into
    dev["o"] and dev["lse"], so only q, k, v and dout cross to the device.
    """
    B, H, N, d = _shape(hq)
    BH = B * H
    hc = max(1, -(-BH // max(1, chunks)))  # heads per group
    caller = torch.cuda.current_stream(dev["q"].device) if stream is None else stream
    s_in = torch.cuda.Stream(device=dev["q"].device)
    s_run = torch.cuda.Stream(device=dev["q"].device)
    s_out = torch.cuda.Stream(device=dev["q"].device)
    start = torch.cuda.Event()
    start.record(caller)
    for s in (s_in, s_run, s_out):
        s.wait_event(start)

    def rows(t):  # [B, H, ...] -> [B*H, ...]
        return t.reshape(BH, *t.shape[2:])

    names = ("q", "k", "v", "dout") if recompute_forward else ("q", "k", "v", "o", "dout", "lse")
    hosts = dict(zip(("q", "k", "v", "o", "dout", "lse"), (hq, hk, hv, ho, hdout, hlse)))
    outs = (("dq", hdq), ("dk", hdk), ("dv", hdv))
    done = None
    for c0 in range(0, BH, hc):
        c1 = min(BH, c0 + hc)
        with torch.cuda.stream(s_in):
            for n in names:
                rows(dev[n])[c0:c1].copy_(rows(hosts[n])[c0:c1], non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(s_in)
        s_run.wait_event(landed)
        view = {n: rows(dev[n])[c0:c1].unsqueeze(0)
                for n in ("q", "k", "v", "o", "dout", "lse", "dq", "dk", "dv")}
        if recompute_forward:
            if block_mask is None:
                attn_fwd(view["q"], view["k"], view["v"], view["o"], view["lse"], causal, scale,
                         s_run)
            else:
                attn_fwd_masked(view["q"], view["k"], view["v"], view["o"], view["lse"],
                                block_mask, scale, s_run)
        if block_mask is None:
            attn_bwd(view["q"], view["k"], view["v"], view["o"], view["dout"], view["lse"],
                     view["dq"], view["dk"], view["dv"], dev["workspace"], causal, scale, s_run)
        else:
            attn_bwd_masked(view["q"], view["k"], view["v"], view["o"], view["dout"], view["lse"],
                            view["dq"], view["dk"], view["dv"], block_mask, dev["workspace"],
                            scale, s_run)
        ready = torch.cuda.Event()
        ready.record(s_run)
        s_out.wait_event(ready)
        with torch.cuda.stream(s_out):
            for n, h in outs:
                rows(h)[c0:c1].copy_(rows(dev[n])[c0:c1], non_blocking=True)
        done = torch.cuda.Event()
        done.record(s_out)
    caller.wait_event(done)


def chunk_workspace_bytes(B: int, H: int, N: int, d: int, dtype, chunks: int = 8) -> int:
    """Workspace bytes for one group of backward_host (the largest group)."""
    hc = max(1, -(-(B * H) // max(1, chunks)))
    return attn_bwd_workspace_bytes(1, hc, N, d, dtype)


def block_mask_tiles(N: int) -> int:
    """Side of the block mask for N positions: ceil(N / 128) tiles."""
    return -(-N // 128)


def attn_fwd_masked(q, k, v, o, lse, block_mask, scale: float | None = None, stream=None,
                    check: bool = True) -> int:
    """O, LSE <- block-sparse forward; `block_mask` is a CUDA uint8 [T, T]
    tensor of tile kinds (0 none, 1 all, 2 key <= query inside the tile)."""
    B, H, N, d = _shape(q)
    scale = d ** -0.5 if scale is None else scale
    st = _lib.attn_fwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                              _ptr(block_mask), float(scale), _DTYPES[q.dtype], _stream(stream))
    if check:
        _check(st, "attn_fwd_masked")
    return st


def attn_bwd_masked(q, k, v, o, dout, lse, dq, dk, dv, block_mask, workspace,
                    scale: float | None = None, stream=None, check: bool = True) -> int:
    """dQ, dK, dV <- block-sparse backward (same block mask as the forward)."""
    B, H, N, d = _shape(q)
    scale = d ** -0.5 if scale is None else scale
    st = _lib.attn_bwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                              _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, _ptr(block_mask),
                              float(scale), _DTYPES[q.dtype], _ptr(workspace),
                              int(workspace.numel()), _stream(stream))
    if check:
        _check(st, "attn_bwd_masked")
    return st
