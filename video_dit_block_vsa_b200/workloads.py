"""Seeded synthetic workloads shaped like the pages' video-DiT latents.

This module only draws inputs; it holds none of the attention arithmetic, so
both the CUDA path and the CPU oracle may take their inputs from it.

Shapes (latent grid T x H x W, heads, head dim, top-k) follow the workloads the
FastWan / VSA pages name: the 410M scaling DiT on a (16, 32, 32) latent at
87.5 % sparsity, Wan-1.3B finetuned on 16x28x52 latents, Wan-1.3B at 480p
(21x30x52, a grid whose sides are not all multiples of 4) with a top-k ratio of
0.1, and Wan-14B at 720p (21x45x80, more than 80k tokens).  The pages measure on
Wan / Hunyuan latents and VBench; neither is available, and these inputs stand
in for them.

Recipe (all float32 draws from ``numpy.random.default_rng(seed)``, in this
order): q, k, v ~ N(0, 1) of shape [B, H, N, d]; then, when ``cube_mean_std``
is set, for q, k and v in turn one vector m ~ N(0, cube_mean_std^2) in R^d per
(b, h, cube coordinate) is added to every token of that cube, so that cube
scores are non-uniform; then, when gated, g_f and g_c ~ U[0, 1) of shape
[B, H, N].  q, k, v are rounded to bf16 (round to nearest even) and returned as
uint16 bit patterns.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    grid: tuple          # (T, H, W) latent token grid
    topk: int            # selected key cubes per query cube
    seed: int
    cube_mean_std: float  # 0.0: no per-cube mean
    gated: bool

    @property
    def tokens(self) -> int:
        return self.grid[0] * self.grid[1] * self.grid[2]

    @property
    def cubes(self) -> int:
        return math.prod(-(-g // 4) for g in self.grid)


def _k_from_ratio(cubes: int, ratio: float) -> int:
    return max(1, int(math.floor(ratio * cubes + 0.5)))


def _mk(name, B, H, d, grid, seed, std, gated, topk=None, ratio=None):
    C = math.prod(-(-g // 4) for g in grid)
    k = topk if topk is not None else _k_from_ratio(C, ratio)
    return Workload(name, B, H, d, tuple(grid), k, seed, std, gated)


WORKLOADS = {
    w.name: w for w in [
        _mk("tiny_k2", 1, 2, 64, (4, 8, 8), 0, 0.0, True, topk=2),
        _mk("tiny_dense", 1, 2, 64, (4, 8, 8), 0, 0.0, True, topk=4),
        _mk("scaling_16x32x32", 1, 12, 128, (16, 32, 32), 1, 0.5, False, topk=32),
        _mk("wan1.3b_ft_16x28x52", 1, 12, 128, (16, 28, 52), 2, 0.5, True, topk=46),
        _mk("wan1.3b_480p_21x30x52", 1, 12, 128, (21, 30, 52), 3, 0.5, False, ratio=0.1),
        _mk("wan14b_720p_21x45x80_k180", 1, 40, 128, (21, 45, 80), 4, 0.5, False, ratio=0.125),
        _mk("wan14b_720p_21x45x80_k43", 1, 40, 128, (21, 45, 80), 4, 0.5, False, ratio=0.03),
        _mk("wan14b_720p_21x45x80_dense", 1, 40, 128, (21, 45, 80), 4, 0.5, False, ratio=1.0),
    ]
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest even) and return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def make_inputs(w: Workload, heads: int | None = None):
    """Draw the inputs of workload ``w``.

    Returns dict(q, k, v: uint16 bf16 bits [B, H, N, d]; g_f, g_c: float32
    [B, H, N] or None).  ``heads`` limits the draw to the first heads (the
    draw order is per tensor, so a head subset is not a prefix of the full
    draw; use it only for self-contained small checks).
    """
    H = w.heads if heads is None else heads
    B, d = w.batch, w.head_dim
    T, Y, X = w.grid
    N = T * Y * X
    rng = np.random.default_rng(w.seed)
    q = rng.standard_normal((B, H, N, d), dtype=np.float32)
    k = rng.standard_normal((B, H, N, d), dtype=np.float32)
    v = rng.standard_normal((B, H, N, d), dtype=np.float32)
    if w.cube_mean_std > 0.0:
        Ct, Cy, Cx = -(-T // 4), -(-Y // 4), -(-X // 4)
        t_idx = np.arange(T) // 4
        y_idx = np.arange(Y) // 4
        x_idx = np.arange(X) // 4
        for arr in (q, k, v):
            m = rng.standard_normal((B, H, Ct, Cy, Cx, d), dtype=np.float32)
            m *= np.float32(w.cube_mean_std)
            per_token = m[:, :, t_idx][:, :, :, y_idx][:, :, :, :, x_idx]
            arr += per_token.reshape(B, H, N, d)
    g_f = g_c = None
    if w.gated:
        g_f = rng.random((B, H, N), dtype=np.float32)
        g_c = rng.random((B, H, N), dtype=np.float32)
    return dict(q=f32_to_bf16_bits(q), k=f32_to_bf16_bits(k), v=f32_to_bf16_bits(v),
                g_f=g_f, g_c=g_c)
