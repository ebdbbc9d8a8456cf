"""Head-sharded attention over several GPUs, one process per GPU.

Every (batch, head) pair of attention is independent, so a job of B*H heads
splits into contiguous blocks of the flattened head index, one block per
rank: rank r owns heads [start, end) of head_range(B*H, world, r). Each rank
runs the ordinary kernels on its block; nothing crosses between GPUs on the
data path. gather_heads is the one collective, for a caller who needs every
head's result on every rank: an NCCL (or gloo, on CPU) all-gather of the
blocks back into the [B, H, ...] layout.
"""
from __future__ import annotations

import torch


def head_range(BH: int, world: int, rank: int) -> tuple[int, int]:
    """Heads [start, end) of rank `rank`: blocks of ceil(BH / world) heads in
    rank order (the last ranks may get fewer, or none when BH < world)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    per = -(-BH // world)
    start = min(BH, rank * per)
    return start, min(BH, start + per)


def head_block(t: torch.Tensor, start: int, end: int) -> torch.Tensor:
    """Heads [start, end) of a [B, H, ...] tensor with contiguous (batch, head)
    rows, as a [1, end - start, ...] view (no copy)."""
    flat = t.reshape(t.shape[0] * t.shape[1], *t.shape[2:])
    return flat[start:end].unsqueeze(0)


def backward_shard(q, k, v, o, dout, lse, dq, dk, dv, workspace, world: int, rank: int,
                   causal: bool = True, scale: float | None = None, stream=None) -> tuple[int, int]:
    """The backward of this rank's heads, written into its block of dq, dk,
    dv (full-size [B, H, N, d] tensors; other ranks' blocks are untouched).
    `workspace` needs attn_bwd_workspace_bytes(1, end - start, N, d, dtype)
    bytes. Returns the rank's head range."""
    from . import attn_bwd
    B, H = q.shape[0], q.shape[1]
    start, end = head_range(B * H, world, rank)
    if end > start:
        blk = [head_block(t, start, end) for t in (q, k, v, o, dout, lse, dq, dk, dv)]
        attn_bwd(*blk, workspace, causal, scale, stream)
    return start, end


def gather_heads(t: torch.Tensor, world: int, rank: int, group=None) -> torch.Tensor:
    """All-gather every rank's head block of a [B, H, ...] tensor, so that
    each rank holds all of it (the blocks are padded to equal size for the
    collective)."""
    import torch.distributed as dist
    B, H = t.shape[0], t.shape[1]
    BH = B * H
    per = -(-BH // world)
    flat = t.reshape(BH, *t.shape[2:])
    start, end = head_range(BH, world, rank)
    mine = torch.zeros((per,) + tuple(flat.shape[1:]), dtype=t.dtype, device=t.device)
    mine[: end - start] = flat[start:end]
    out = torch.empty((per * world,) + tuple(flat.shape[1:]), dtype=t.dtype, device=t.device)
    dist.all_gather_into_tensor(out, mine, group=group)
    return out[:BH].reshape(t.shape)
