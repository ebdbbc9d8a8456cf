"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This module holds no attention arithmetic: it only draws random tensors (and
builds the deterministic sinusoid input of the ddx issue #217 repro), so that
the float64 oracle and the CUDA library see exactly the same bits.

Draw order and distribution: one ``torch.Generator('cpu')`` seeded with the
config's seed draws q, k, v, dO in that order, each ``randn(B, H, N, d)`` in
float32. q and k are multiplied by ``qk_gain`` (0.5 for the 262,144-token
case, 1.0 otherwise). For bf16 configs the float32 draws are rounded to
bfloat16 (round-to-nearest-even, as ``Tensor.to(torch.bfloat16)`` rounds); the
oracle then widens exactly those rounded values to float64.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class AttnConfig:
    """One workload: shape [B, H, N, d], element type and seed."""

    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str  # "f32" or "bf16"
    seed: int
    qk_gain: float = 1.0
    causal: bool = True

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def bwd_flops(self) -> float:
        """Causal backward FLOPs, counted as 2.5x the causal forward's 4*B*H*N^2*d/2."""
        return 5.0 * self.B * self.H * self.N * self.N * self.d

    @property
    def fwd_flops(self) -> float:
        return 2.0 * self.B * self.H * self.N * self.N * self.d


# The five workloads: a 256-token single head (fp32), the nanoGPT-shaped
# batch of ddx issue #217 (12 sequences, 4 heads, 64 positions, 128 channels),
# 1,024 tokens, 16,384 tokens x 32 heads, and 262,144 tokens (FlashBoB's length).
CONFIGS = {
    "c1": AttnConfig("c1", 1, 1, 256, 64, "f32", 0),
    "c2_f32": AttnConfig("c2_f32", 12, 4, 64, 32, "f32", 1),
    "c2_bf16": AttnConfig("c2_bf16", 12, 4, 64, 32, "bf16", 1),
    "c3": AttnConfig("c3", 1, 1, 1024, 64, "bf16", 2),
    "c4": AttnConfig("c4", 2, 16, 16384, 128, "bf16", 3),
    "c5": AttnConfig("c5", 1, 4, 262144, 64, "bf16", 4, qk_gain=0.5),
    # a quarter of c4 (8 heads): still larger than L2, small enough for a
    # many-pass profiler capture
    "prof_d128": AttnConfig("prof_d128", 1, 8, 16384, 128, "bf16", 5),
    # the d = 64 counterpart (the long-sequence workload's head size), with
    # its q, k scaling; 8 heads of 32,768 tokens
    "prof_d64": AttnConfig("prof_d64", 1, 8, 32768, 64, "bf16", 6, qk_gain=0.5),
    # backward-over-backward at a length where its fp32 kernels fill the GPU
    "bob_4k": AttnConfig("bob_4k", 1, 8, 4096, 64, "f32", 7),
    # the bf16 tensor-core backward-over-backward at 16,384 tokens, d = 64 and 128
    "bob_16k": AttnConfig("bob_16k", 1, 8, 16384, 64, "bf16", 8),
    "bob_16k_d128": AttnConfig("bob_16k_d128", 1, 4, 16384, 128, "bf16", 9),
}


def draw(B: int, H: int, N: int, d: int, seed: int, dtype: str = "f32",
         qk_gain: float = 1.0):
    """Return q, k, v, dO as CPU tensors of ``dtype`` ('f32' or 'bf16')."""
    g = torch.Generator("cpu").manual_seed(seed)
    out = []
    for name in ("q", "k", "v", "do"):
        t = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
        if name in ("q", "k") and qk_gain != 1.0:
            t = t * qk_gain
        out.append(t.to(torch.bfloat16) if dtype == "bf16" else t)
    return tuple(out)


def draw_rect(B: int, H: int, n_q: int, n_k: int, d: int, seed: int, dtype: str = "f32"):
    """q, k, v, dO for N_q query rows and N_k keys: one seeded CPU generator
    draws q [B, H, N_q, d], k, v [B, H, N_k, d] and dO [B, H, N_q, d] in that
    order, N(0, 1) float32, rounded like `draw` for bf16."""
    g = torch.Generator("cpu").manual_seed(seed)
    out = []
    for n in (n_q, n_k, n_k, n_q):
        t = torch.randn(B, H, n, d, generator=g, dtype=torch.float32)
        out.append(t.to(torch.bfloat16) if dtype == "bf16" else t)
    return tuple(out)


def draw_config(cfg: AttnConfig):
    return draw(cfg.B, cfg.H, cfg.N, cfg.d, cfg.seed, cfg.dtype, cfg.qk_gain)


def as_f64(t: torch.Tensor) -> np.ndarray:
    """Widen a CPU tensor (f32 or bf16) to a float64 numpy array, exactly."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def ddx_issue217_input(S: int = 3, T: int = 8, H: int = 2, C: int = 4):
    """The deterministic repro input of ddx issue #217.

    q, k, v hold sin(n * 0.37 + phase) for n = 0 .. S*T*H*C-1 in (seq, pos,
    head, channel) order, with phase 0, 1, 2. Returned as float64 arrays
    permuted to this library's [B, H, N, d] layout (B = seq, N = pos).
    """
    n = np.arange(S * T * H * C, dtype=np.float64)
    outs = []
    for phase in (0.0, 1.0, 2.0):
        x = np.sin(n * 0.37 + phase).reshape(S, T, H, C)
        outs.append(np.ascontiguousarray(x.transpose(0, 2, 1, 3)))
    return tuple(outs)


# ----------------------------------------------------------------- block masks
# Tile kinds of a block mask over 128 x 128 tiles: 0 the tile takes no part,
# 1 every score of the tile takes part, 2 a score takes part when its key's
# index inside the tile is at most its query's.
TILE = 128


def block_mask(spec: str, N: int) -> np.ndarray:
    """A [T, T] uint8 block mask (T = ceil(N / 128)) named by `spec`:

    * ``causal``: kind 2 on the diagonal, 1 below it (the causal mask, tile by tile);
    * ``full``: every tile kind 1;
    * ``window:W``: local causal attention over W tiles: query tile i sees key
      tiles i-W+1 .. i-1 in full and its own tile causally;
    * ``random:P:SEED``: the causal mask with each below-diagonal tile kept
      with probability P (seeded numpy draw), the diagonal always kept.
    """
    T = -(-N // TILE)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    name, *rest = spec.split(":")
    if name == "causal":
        m = np.where(j < i, 1, np.where(j == i, 2, 0))
    elif name == "full":
        m = np.ones((T, T), dtype=np.int64)
    elif name == "window":
        w = int(rest[0])
        if w < 1:
            raise ValueError("window needs W >= 1")
        m = np.where(j == i, 2, np.where((j < i) & (j > i - w), 1, 0))
    elif name == "random":
        p, seed = float(rest[0]), int(rest[1]) if len(rest) > 1 else 0
        keep = np.random.default_rng(seed).random((T, T)) < p
        m = np.where(j == i, 2, np.where((j < i) & keep, 1, 0))
    else:
        raise ValueError(f"unknown block mask {spec!r}")
    return np.ascontiguousarray(m.astype(np.uint8))


def block_mask_pairs(mask: np.ndarray) -> float:
    """Score pairs a block mask keeps, counted the causal way: a kind-1 tile
    as 128 * 128 pairs, a kind-2 tile as half of that (so the causal mask of
    N = 128 T positions counts N^2 / 2)."""
    m = np.asarray(mask)
    return float(TILE * TILE * (np.count_nonzero(m == 1) + 0.5 * np.count_nonzero(m == 2)))


def draw_layer(B: int, N: int, C: int, seed: int, dtype: str = "bf16"):
    """Inputs of one attention layer: x, dy ~ N(0, 1) [B, N, C] and weights
    W_qkv [C, 3C], W_o [C, C] ~ N(0, 1/C), drawn in that order from one seeded
    CPU generator (float32, then rounded like `draw`)."""
    g = torch.Generator("cpu").manual_seed(seed)
    x = torch.randn(B, N, C, generator=g)
    w_qkv = torch.randn(C, 3 * C, generator=g) / math.sqrt(C)
    w_o = torch.randn(C, C, generator=g) / math.sqrt(C)
    dy = torch.randn(B, N, C, generator=g)
    if dtype == "bf16":
        x, w_qkv, w_o, dy = (t.to(torch.bfloat16) for t in (x, w_qkv, w_o, dy))
    return x, w_qkv, w_o, dy
