"""Sequence-parallel SQuad-Attention forward over G ranks (one process per GPU).

Rank r holds the tokens of a contiguous range of whole frame windows of the
T x H x W grid. The local pass needs nothing from other ranks; for the global
pass one all-to-all moves Q, K and the local-pass output from window-major to
position-major (each rank then holds, for its share of the in-window positions,
one row of every window), the global pass runs on that layout, and a second
all-to-all returns the output rows to their owners. The layout, the index maps
and the shuffle kernels are the library's (squad_sp_* in include/squad.h); this
module marshals arguments and issues the two collectives through
torch.distributed (NCCL on GPUs).
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np
import torch

from . import SquadDesc, _check, _check_inputs, _ptr, _stream_handle, load_library, squad_attn_fwd_pass

__all__ = ["SpPlan", "sp_attention_fwd", "sp_pack", "sp_unpack"]

_INT_P = ctypes.POINTER(ctypes.c_int)


def _lib():
    lib = load_library()
    if not getattr(lib, "_sp_ready", False):
        dp = ctypes.POINTER(SquadDesc)
        vp = ctypes.c_void_p
        lib.squad_sp_plan_info.argtypes = [dp, ctypes.c_int, ctypes.c_int, _INT_P]
        lib.squad_sp_plan_maps.argtypes = [dp, ctypes.c_int, ctypes.c_int] + [_INT_P] * 7
        lib.squad_sp_pack.argtypes = [ctypes.POINTER(vp), ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, _INT_P, vp, vp, vp]
        lib.squad_sp_unpack.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        _INT_P, vp, vp, ctypes.POINTER(vp), vp]
        for f in ("squad_sp_plan_info", "squad_sp_plan_maps", "squad_sp_pack", "squad_sp_unpack"):
            getattr(lib, f).restype = ctypes.c_int
        lib._sp_ready = True
    return lib


def _ints(a: np.ndarray):
    return a.ctypes.data_as(_INT_P)


class SpPlan:
    """Shard layout and index maps of one rank (host arrays; device copies made on first use).

    grid, tile: the whole problem's T x H x W grid and window tile; G ranks.
    Attributes: t0, T (this rank's frames), n_local (its tokens), n_pos (its
    position-major rows), p0, np_ (its positions), w, m, and the maps and
    per-peer row counts of squad_sp_plan_maps.
    """

    def __init__(self, B: int, heads: int, d: int, grid: Sequence[int], tile: Sequence[int], G: int, rank: int,
                 dtype: torch.dtype = torch.bfloat16, scale: Optional[float] = None):
        lib = _lib()
        T, H, W = (int(x) for x in grid)
        tT, tH, tW = (int(x) for x in tile)
        code = 1 if dtype == torch.bfloat16 else 0
        self.desc = SquadDesc(B, heads, d, T, H, W, tT, tH, tW, code, float(scale or 0.0))
        info = (ctypes.c_int * 8)()
        _check(lib.squad_sp_plan_info(ctypes.byref(self.desc), G, rank, info), "squad_sp_plan_info")
        self.t0, self.T, self.n_local, self.n_pos, self.p0, self.np_, self.w, self.m = list(info)
        self.G, self.rank, self.B, self.heads, self.d = G, rank, B, heads, d
        self.grid, self.tile, self.scale = (T, H, W), (tT, tH, tW), scale
        self.counts = np.zeros(4 * G, dtype=np.int32)
        self.send1 = np.zeros(self.n_local, dtype=np.int32)
        self.recv1_src = np.zeros(self.n_pos, dtype=np.int32)
        self.recv1_row = np.zeros(self.n_pos, dtype=np.int32)
        self.send2 = np.zeros(self.n_pos, dtype=np.int32)
        self.recv2_src = np.zeros(self.n_local, dtype=np.int32)
        self.recv2_row = np.zeros(self.n_local, dtype=np.int32)
        _check(lib.squad_sp_plan_maps(ctypes.byref(self.desc), G, rank, _ints(self.counts), _ints(self.send1),
                                      _ints(self.recv1_src), _ints(self.recv1_row), _ints(self.send2),
                                      _ints(self.recv2_src), _ints(self.recv2_row)), "squad_sp_plan_maps")
        self.send1_count, self.recv1_count, self.send2_count, self.recv2_count = (
            self.counts[i * G:(i + 1) * G].copy() for i in range(4))
        self._dev = {}

    # the local pass on this rank's shard, the global pass on its position-major rows
    @property
    def local_grid(self):
        return (self.T,) + self.grid[1:]

    @property
    def global_grid(self):
        T, H, W = self.grid
        tT, tH, tW = self.tile
        return (self.np_ * (T // tT), H // tH, W // tW)

    @property
    def global_tile(self):
        T, H, W = self.grid
        tT, tH, tW = self.tile
        return (T // tT, H // tH, W // tW)

    def device_maps(self, device: torch.device):
        key = str(device)
        if key not in self._dev:
            self._dev[key] = {n: torch.from_numpy(getattr(self, n)).to(device)
                              for n in ("send1", "recv1_src", "recv1_row", "send2", "recv2_src", "recv2_row")}
        return self._dev[key]


def sp_pack(srcs: Sequence[torch.Tensor], idx: torch.Tensor, counts: np.ndarray, stream=None) -> torch.Tensor:
    """Rows of srcs (each [B, h, rows_in, d]) in the exchange layout [peer][tensor][slice][counts[peer]]."""
    lib = _lib()
    _check_inputs(*srcs)
    B, h, rows_in, d = srcs[0].shape
    slices = B * h
    if not (1 <= len(srcs) <= 3):
        raise ValueError("one to three source tensors")
    if idx.dtype != torch.int32 or not idx.is_cuda or idx.device != srcs[0].device or idx.numel() != int(counts.sum()):
        raise ValueError("idx must be a device int32 tensor with one entry per packed row")
    total = int(counts.sum()) * len(srcs) * slices
    out = torch.empty((total, d), device=srcs[0].device, dtype=srcs[0].dtype)
    ptrs = (ctypes.c_void_p * len(srcs))(*[t.data_ptr() for t in srcs])
    c = np.ascontiguousarray(counts, dtype=np.int32)
    with torch.cuda.device(srcs[0].device):
        _check(lib.squad_sp_pack(ptrs, len(srcs), slices, rows_in, d * srcs[0].element_size(), len(c), _ints(c),
                                 _ptr(idx), _ptr(out), _stream_handle(stream, srcs[0].device)), "squad_sp_pack")
    return out


def sp_unpack(src: torch.Tensor, ntensors: int, B: int, h: int, rows_out: int, src_rank: torch.Tensor,
              src_row: torch.Tensor, counts: np.ndarray, stream=None):
    """The inverse layout change: ntensors tensors [B, h, rows_out, d] gathered from src."""
    lib = _lib()
    d = src.shape[-1]
    for t in (src_rank, src_row):
        if t.dtype != torch.int32 or not t.is_cuda or t.device != src.device or t.numel() != rows_out:
            raise ValueError("src_rank and src_row must be device int32 tensors of rows_out entries")
    if not src.is_cuda or src.dim() != 2 or src.shape[0] != int(counts.sum()) * ntensors * B * h:
        raise ValueError("src must be the [rows, d] exchange buffer of these counts")
    outs = [torch.empty((B, h, rows_out, d), device=src.device, dtype=src.dtype) for _ in range(ntensors)]
    ptrs = (ctypes.c_void_p * ntensors)(*[t.data_ptr() for t in outs])
    c = np.ascontiguousarray(counts, dtype=np.int32)
    with torch.cuda.device(src.device):
        _check(lib.squad_sp_unpack(_ptr(src), ntensors, B * h, rows_out, d * src.element_size(), len(c), _ints(c),
                                   _ptr(src_rank), _ptr(src_row), ptrs, _stream_handle(stream, src.device)),
               "squad_sp_unpack")
    return outs


def _split(counts: np.ndarray, ntensors: int, slices: int):
    return [int(x) * ntensors * slices for x in counts]


def sp_attention_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, plan: SpPlan, group=None) -> torch.Tensor:
    """SQuad-Attention forward of this rank's shard ([B, h, n_local, d] CUDA tensors, tokens of
    frames [plan.t0, plan.t0 + plan.T)); returns the output rows of the same tokens.

    Collective: every rank of `group` (world size plan.G) calls it with the same plan shape.
    """
    import torch.distributed as dist
    _check_inputs(q, k, v)
    B, h, n_local, d = q.shape
    if n_local != plan.n_local or (B, h, d) != (plan.B, plan.heads, plan.d):
        raise ValueError("shard shape does not match the plan")
    maps = plan.device_maps(q.device)
    slices = B * h
    # local pass on this rank's windows
    o1 = torch.empty_like(q)
    squad_attn_fwd_pass(1, q, k, v, o1, plan.local_grid, plan.tile, plan.scale)
    # window-major -> position-major: Q, K and the local-pass output
    send = sp_pack([q, k, o1], maps["send1"], plan.send1_count)
    recv = torch.empty((int(plan.recv1_count.sum()) * 3 * slices, d), device=q.device, dtype=q.dtype)
    dist.all_to_all_single(recv, send, _split(plan.recv1_count, 3, slices), _split(plan.send1_count, 3, slices),
                           group=group)
    qg, kg, o1g = sp_unpack(recv, 3, B, h, plan.n_pos, maps["recv1_src"], maps["recv1_row"], plan.recv1_count)
    # global pass: each window of the position-major grid is one group
    og = torch.empty_like(qg)
    squad_attn_fwd_pass(1, qg, kg, o1g, og, plan.global_grid, plan.global_tile, plan.scale)
    # and back to the owners' token order
    send2 = sp_pack([og], maps["send2"], plan.send2_count)
    recv2 = torch.empty((int(plan.recv2_count.sum()) * slices, d), device=q.device, dtype=q.dtype)
    dist.all_to_all_single(recv2, send2, _split(plan.recv2_count, 1, slices), _split(plan.send2_count, 1, slices),
                           group=group)
    (o,) = sp_unpack(recv2, 1, B, h, plan.n_local, maps["recv2_src"], maps["recv2_row"], plan.recv2_count)
    return o
