"""Seeded synthetic inputs for the SQuad-Attention workloads.

This module only draws random numbers and holds the workload shapes. It holds
none of the method's arithmetic, so both the fp64 oracle (``oracle/``) and the
CUDA path (``sub_quadratic_two_b200``) can be fed from it without sharing code.

The shapes stand in for the attention of a Wan 2.2 5B text-to-video DiT block
(24 heads, head dim 128, latent grid 31x22x40), the workload of the results
section of "SQuad: Sub-Quadratic Attention Distillation for Efficient Video
Generation" (gist.science technical summary, Experimental Results). The pages
give neither the data nor the trained weights, so every tensor is synthetic.

Recipe (all workloads): a CPU ``torch.Generator`` seeded with the workload's
seed draws, in this order and in fp32, ``randn`` tensors for Q, K, V [B, h, n, d]
and then the workload's extra terms; the result is cast to the workload dtype.
The cast tensors are the ground truth handed to both sides.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    dtype: str            # "f32" or "bf16"
    B: int
    heads: int
    d: int
    grid: Tuple[int, int, int]   # (T, H, W)
    tile: Tuple[int, int, int]   # (tT, tH, tW)
    k_bias_std: float = 0.0      # shared per-channel K bias b ~ N(0, std^2), one vector for all rows
    head_scale: Optional[Tuple[float, float]] = None  # sigma_h ~ U[lo, hi] scales Q and K of head h
    backward: bool = False       # also draw the upstream gradient dO
    note: str = ""

    @property
    def n(self) -> int:
        T, H, W = self.grid
        return T * H * W

    @property
    def w(self) -> int:
        tT, tH, tW = self.tile
        return tT * tH * tW

    @property
    def m(self) -> int:
        return self.n // self.w

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def fwd_flops(self) -> float:
        """Useful forward FLOPs, 4*n*d*(w+m) per (batch, head)."""
        return 4.0 * self.n * self.d * (self.w + self.m) * self.B * self.heads

    def bwd_flops(self) -> float:
        """Useful backward FLOPs: five GEMMs per stage, 2.5x the forward."""
        return 2.5 * self.fwd_flops()

    def dense_flops(self) -> float:
        return 4.0 * self.n * self.n * self.d * self.B * self.heads


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_fp32", 1, "f32", 1, 2, 64, (4, 8, 8), (1, 4, 4),
                 note="n=256, w=16, m=16; Q,K,V ~ N(0,1)"),
        Workload("small_bf16", 2, "bf16", 1, 8, 128, (8, 16, 16), (2, 4, 8), k_bias_std=2.0,
                 note="n=2048, w=64, m=32; K gets a shared per-channel bias N(0,2^2)"),
        Workload("wan5b_fwd", 3, "bf16", 1, 24, 128, (31, 22, 40), (1, 11, 20), head_scale=(0.5, 2.0),
                 note="n=27280, w=220, m=124; Q,K scaled per head by U[0.5,2]"),
        Workload("wan5b_train", 4, "bf16", 2, 24, 128, (31, 22, 40), (1, 11, 20), backward=True,
                 note="forward + backward, dO ~ N(0,1)"),
        Workload("long_video", 5, "bf16", 1, 24, 128, (61, 22, 40), (1, 22, 20), k_bias_std=2.0,
                 note="n=53680, w=440, m=122; K gets a shared per-channel bias N(0,2^2)"),
    ]
}


@dataclass
class Inputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    do: Optional[torch.Tensor] = None
    extras: Dict[str, torch.Tensor] = field(default_factory=dict)


def make_inputs(wl: Workload, seed: Optional[int] = None, heads: Optional[int] = None) -> Inputs:
    """Draw the workload's inputs on the CPU (see the module docstring for the order).

    ``heads`` overrides the head count (used for cut-down parity cases); the draw
    order is unchanged, so a run with fewer heads is a different sample.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed if seed is None else seed)
    h = wl.heads if heads is None else heads
    shape = (wl.B, h, wl.n, wl.d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    extras: Dict[str, torch.Tensor] = {}
    if wl.k_bias_std:
        b = torch.randn((wl.d,), generator=g, dtype=torch.float32) * wl.k_bias_std
        k = k + b
        extras["k_bias"] = b
    if wl.head_scale is not None:
        lo, hi = wl.head_scale
        sig = lo + (hi - lo) * torch.rand((h,), generator=g, dtype=torch.float32)
        q = q * sig.view(1, h, 1, 1)
        k = k * sig.view(1, h, 1, 1)
        extras["head_scale"] = sig
    do = None
    if wl.backward:
        do = torch.randn(shape, generator=g, dtype=torch.float32)
    dt = wl.torch_dtype
    return Inputs(q.to(dt), k.to(dt), v.to(dt), None if do is None else do.to(dt), extras)


def random_problem(seed: int, B: int, heads: int, d: int, grid, tile, dtype=torch.float32,
                   k_bias_std: float = 0.0, with_do: bool = False) -> Inputs:
    """Generic seeded case for tests: Q, K, V (and dO) ~ N(0,1) [B, heads, T*H*W, d]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    n = grid[0] * grid[1] * grid[2]
    shape = (B, heads, n, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    if k_bias_std:
        k = k + torch.randn((d,), generator=g, dtype=torch.float32) * k_bias_std
    do = torch.randn(shape, generator=g, dtype=torch.float32) if with_do else None
    return Inputs(q.to(dtype), k.to(dtype), v.to(dtype), None if do is None else do.to(dtype))
