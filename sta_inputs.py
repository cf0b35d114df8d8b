"""Seeded synthetic workloads for Sliding Tile Attention.

This module only draws inputs.  It holds none of the method's arithmetic (no
masks, no tile lists, no attention), so both the CUDA path and the CPU oracle
can take their inputs from it without sharing any computation.

The workloads stand in for HunyuanVideo 720p 5 s attention activations (the
pages measure STA on that model; its weights and prompts are not available),
with the latent shapes, head counts, head dimension, tile and windows of the
five configurations below.  Values are i.i.d. N(0, 1) drawn in fp32 and rounded
to bf16 (round to nearest even), optionally multiplied per head by a factor
f_h ~ U[0.5, 2] before the rounding (configuration 5).

Every (configuration, tensor, batch, head) slice has its own seed (numpy
PCG64 stream), so any slice can be regenerated alone: the oracle only draws the
heads it samples.  Slices are drawn on a thread pool.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np
import torch

TILE = (6, 8, 8)

# Windows (tokens) named on the pages: (18,24,24) and (30,40,40) are the STA
# windows evaluated on HunyuanVideo; (30,48,80) covers the whole 720p latent.
W_SMALL = (18, 24, 24)
W_MID = (30, 40, 40)
W_FULL_720P = (30, 48, 80)


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    batch: int
    heads: int
    head_dim: int
    latent: tuple
    tile: tuple
    window: tuple | None  # one window for every head, or None when drawn per head
    head_factors: bool = False

    @property
    def tokens(self) -> int:
        return self.latent[0] * self.latent[1] * self.latent[2]

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def seed(self) -> int:
        return 1000 + self.index


WORKLOADS = {
    1: Workload(1, "tiny_18x24x24_w12x16x16", 1, 2, 64, (18, 24, 24), TILE, (12, 16, 16)),
    2: Workload(2, "720p_30x48x80_w18x24x24", 1, 24, 128, (30, 48, 80), TILE, W_SMALL),
    3: Workload(3, "720p_30x48x80_mixed_per_head", 1, 24, 128, (30, 48, 80), TILE, None),
    4: Workload(4, "720p_30x48x80_full_window", 1, 24, 128, (30, 48, 80), TILE, W_FULL_720P),
    5: Workload(5, "large_42x64x112_w30x40x40_scaled", 2, 24, 128, (42, 64, 112), TILE, W_MID,
                head_factors=True),
}

MIXED_CHOICES = (W_SMALL, W_MID, W_FULL_720P)


def windows(w: Workload) -> torch.Tensor:
    """``[heads, 3]`` int32 window per head, in tokens."""
    if w.window is not None:
        return torch.tensor([list(w.window)] * w.heads, dtype=torch.int32)
    idx = np.random.default_rng(w.seed).integers(0, len(MIXED_CHOICES), size=w.heads)
    return torch.tensor([list(MIXED_CHOICES[i]) for i in idx.tolist()], dtype=torch.int32)


def head_factors(w: Workload) -> torch.Tensor | None:
    """Per-head factor f_h ~ U[0.5, 2] (fp32) or None."""
    if not w.head_factors:
        return None
    f = np.random.default_rng(w.seed * 7 + 1).uniform(0.5, 2.0, size=w.heads)
    return torch.from_numpy(f.astype(np.float32))


def slice_seed(w: Workload, which: int, b: int, h: int) -> int:
    """Seed of one [N, d] slice; which = 0 (Q), 1 (K), 2 (V), 3 (dO)."""
    return ((w.seed * 4 + which) * 1024 + b) * 1024 + h


def make_slice(w: Workload, which: int, b: int, h: int) -> torch.Tensor:
    """One ``[N, d]`` bf16 slice (CPU), raster token order."""
    rng = np.random.default_rng(slice_seed(w, which, b, h))
    x = torch.from_numpy(rng.standard_normal((w.tokens, w.head_dim), dtype=np.float32))
    f = head_factors(w)
    if f is not None and which < 3:
        x.mul_(float(f[h]))
    return x.to(torch.bfloat16)


def make_qkv(w: Workload, device="cpu", heads=None, batches=None):
    """Q, K, V as ``[B, H, N, d]`` bf16 tensors on ``device`` (raster order).

    ``heads`` / ``batches`` restrict which slices are drawn (others stay zero),
    for oracle runs that only need a few heads.
    """
    shape = (w.batch, w.heads, w.tokens, w.head_dim)
    out = [torch.zeros(shape, dtype=torch.bfloat16, device=device) for _ in range(3)]
    hs = range(w.heads) if heads is None else heads
    bs = range(w.batch) if batches is None else batches
    jobs = [(which, b, h) for which in range(3) for b in bs for h in hs]

    def one(job):
        which, b, h = job
        out[which][b, h].copy_(make_slice(w, which, b, h))

    with ThreadPoolExecutor(max_workers=max(1, min(16, os.cpu_count() or 1))) as ex:
        list(ex.map(one, jobs))
    return tuple(out)


def make_dout(w: Workload, device="cpu", heads=None, batches=None) -> torch.Tensor:
    """Upstream gradient dO for the backward pass: ``[B, H, N, d]`` bf16, raster
    order, i.i.d. N(0, 1) rounded to bf16 (no head factor), same slice seeding."""
    out = torch.zeros((w.batch, w.heads, w.tokens, w.head_dim), dtype=torch.bfloat16, device=device)
    hs = range(w.heads) if heads is None else heads
    bs = range(w.batch) if batches is None else batches
    jobs = [(b, h) for b in bs for h in hs]

    def one(job):
        b, h = job
        out[b, h].copy_(make_slice(w, 3, b, h))

    with ThreadPoolExecutor(max_workers=max(1, min(16, os.cpu_count() or 1))) as ex:
        list(ex.map(one, jobs))
    return out
