"""fp64 CPU oracle for SQuad-Attention (plain C, loaded through ctypes).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg may use it; the product path never does. It shares no code with
the CUDA library and imports nothing from it.

Parity pins (tests/test_oracle_pins.py): every function here is checked
against facts that do not come from this file -- dense attention from
torch's SDPA when one window covers the grid or every window is one token,
the same two passes written as block-masked dense attention in numpy,
constant-value rows, permutation equivariance, key-shift invariance, the
closed-form multiply-add count 2*n*d*(w+m), a hand-derived two-token case
(tests/golden/), and central finite differences for the backward. The
k-pass functions (passes over nested tiles) are pinned by their reductions
to the two-pass oracle and to dense attention when tiles are trivial, by
three block-masked dense attentions composed in numpy, by their closed-form
multiply-add count, and by finite differences.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "squad_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


class _Desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("heads", ctypes.c_int), ("d", ctypes.c_int),
                ("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("tT", ctypes.c_int), ("tH", ctypes.c_int), ("tW", ctypes.c_int),
                ("scale", ctypes.c_double)]


def build(force: bool = False) -> str:
    """Compile squad_oracle.c into liboracle.so next to it (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_fwd.argtypes = [ctypes.POINTER(_Desc), dp, dp, dp, dp, dp, dp, dp,
                                   ctypes.c_int, ctypes.POINTER(ctypes.c_ulonglong)]
        lib.oracle_fwd.restype = ctypes.c_int
        lib.oracle_bwd.argtypes = [ctypes.POINTER(_Desc), dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
        lib.oracle_bwd.restype = ctypes.c_int
        ip = ctypes.POINTER(ctypes.c_int)
        lib.oracle_fwd_multi.argtypes = [ctypes.POINTER(_Desc), ctypes.c_int, ip, dp, dp, dp, dp, dp, dp,
                                         ctypes.c_int, ctypes.POINTER(ctypes.c_ulonglong)]
        lib.oracle_fwd_multi.restype = ctypes.c_int
        lib.oracle_bwd_multi.argtypes = [ctypes.POINTER(_Desc), ctypes.c_int, ip, dp, dp, dp, dp, dp, dp, dp,
                                         ctypes.c_int]
        lib.oracle_bwd_multi.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _desc(shape, grid, tile, scale) -> _Desc:
    B, h, n, d = shape
    T, H, W = grid
    if T * H * W != n:
        raise ValueError(f"n={n} != T*H*W={T * H * W}")
    return _Desc(B, h, d, T, H, W, tile[0], tile[1], tile[2], float(scale or 0.0))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


def squad_fwd(q, k, v, grid: Tuple[int, int, int], tile: Tuple[int, int, int],
              scale: Optional[float] = None, threads: Optional[int] = None):
    """Two-pass SQuad-Attention forward in fp64.

    Returns (o, o1, lse1, lse2, macs): o and o1 are [B,h,n,d], lse1/lse2 are
    [B,h,n] (natural log), macs is the number of multiply-adds performed.
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    desc = _desc(q.shape, grid, tile, scale)
    o = np.empty_like(q)
    o1 = np.empty_like(q)
    lse1 = np.empty(q.shape[:3])
    lse2 = np.empty(q.shape[:3])
    macs = ctypes.c_ulonglong(0)
    rc = lib.oracle_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(o1),
                        _ptr(lse1), _ptr(lse2), int(threads or default_threads()), ctypes.byref(macs))
    if rc != 0:
        raise ValueError(f"oracle_fwd failed with code {rc}")
    return o, o1, lse1, lse2, int(macs.value)


def squad_bwd(q, k, v, dout, grid, tile, scale: Optional[float] = None, threads: Optional[int] = None):
    """Gradients (dq, dk, dv) of sum(O * dout) through both passes, fp64."""
    lib = _load()
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    desc = _desc(q.shape, grid, tile, scale)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    rc = lib.oracle_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(dout),
                        _ptr(dq), _ptr(dk), _ptr(dv), int(threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_bwd failed with code {rc}")
    return dq, dk, dv


def _tiles(tiles):
    flat = [int(x) for t in tiles for x in t]
    if not tiles or any(len(t) != 3 for t in tiles):
        raise ValueError("tiles: a non-empty list of (tT, tH, tW)")
    return len(tiles), (ctypes.c_int * len(flat))(*flat)


def squad_fwd_multi(q, k, v, grid, tiles, scale: Optional[float] = None, threads: Optional[int] = None):
    """Forward of k = len(tiles) + 1 passes over nested tiles (innermost first), fp64.

    Returns (o, inter, lse, macs): inter is [k-1, B,h,n,d] (outputs of passes
    1..k-1), lse is [k, B,h,n], macs the multiply-adds performed.
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    desc = _desc(q.shape, grid, tiles[0], scale)
    nt, tarr = _tiles(tiles)
    o = np.empty_like(q)
    inter = np.empty((nt,) + q.shape)
    lse = np.empty((nt + 1,) + q.shape[:3])
    macs = ctypes.c_ulonglong(0)
    rc = lib.oracle_fwd_multi(ctypes.byref(desc), nt, tarr, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(inter),
                              _ptr(lse), int(threads or default_threads()), ctypes.byref(macs))
    if rc != 0:
        raise ValueError(f"oracle_fwd_multi failed with code {rc}")
    return o, inter, lse, int(macs.value)


def squad_bwd_multi(q, k, v, dout, grid, tiles, scale: Optional[float] = None, threads: Optional[int] = None):
    """Gradients (dq, dk, dv) of sum(O * dout) through the k passes, fp64."""
    lib = _load()
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    desc = _desc(q.shape, grid, tiles[0], scale)
    nt, tarr = _tiles(tiles)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    rc = lib.oracle_bwd_multi(ctypes.byref(desc), nt, tarr, _ptr(q), _ptr(k), _ptr(v), _ptr(dout),
                              _ptr(dq), _ptr(dk), _ptr(dv), int(threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_bwd_multi failed with code {rc}")
    return dq, dk, dv
