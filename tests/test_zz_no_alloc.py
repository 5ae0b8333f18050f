"""squad_attn_fwd_noalloc: the forward that makes the library allocate nothing.

Some callers cannot hand the library device memory for scratch -- a host
framework that owns every device allocation through its own pool, or
latency-critical code that must not call cudaMalloc because it can
synchronise the device. For them the local-pass output lives in a fixed
32 MiB array inside libsquad. These tests call that entry point through the C
ABI and check it against squad_attn_fwd (which keeps the local-pass output in
caller memory) on two calls in a row, so that a second call reading the first
call's leftovers in the shared array would be caught. This file is collected
last on purpose: a failure here does not hide any other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import sub_quadratic_two_b200 as sq
from workloads import WORKLOADS, make_inputs, random_problem

pytestmark = pytest.mark.gpu

BF16_MAX, BF16_MEAN, LSE_TOL, F32_TOL = 1.5e-2, 2e-3, 2e-3, 1e-5
SCRATCH_BYTES = 32 << 20


def _abi():
    lib = sq.load_library()
    fn = lib.squad_attn_fwd_noalloc
    fn.argtypes = [ctypes.POINTER(sq.SquadDesc)] + [ctypes.c_void_p] * 7
    fn.restype = ctypes.c_int
    return fn


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _inputs(name, second):
    wl = WORKLOADS[name]
    if not second:
        return wl, make_inputs(wl)
    dt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    return wl, random_problem(97, wl.B, wl.heads, wl.d, wl.grid, wl.tile, dtype=dt, k_bias_std=1.0)


def _close(a, b, fp32, what):
    e = (a.double() - b.double()).abs()
    assert torch.isfinite(a).all(), what
    if fp32:
        assert e.max().item() <= F32_TOL, (what, e.max().item())
    else:
        assert e.max().item() <= BF16_MAX and e.mean().item() <= BF16_MEAN, (what, e.max().item(), e.mean().item())


@pytest.mark.parametrize("name", ["small_bf16", "tiny_fp32"])
def test_noalloc_matches_forward_on_two_calls_in_a_row(cuda_ok, name):
    fn = _abi()
    cases = []
    for second in (False, True):
        wl, inp = _inputs(name, second)
        q, k, v = (t.cuda().contiguous() for t in (inp.q, inp.k, inp.v))
        ref_o, _, ref_l1, ref_l2 = sq.squad_attn_fwd(q, k, v, wl.grid, wl.tile, save=True)
        cases.append((wl, q, k, v, ref_o, ref_l1, ref_l2))
    torch.cuda.synchronize()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    outs = []
    for wl, q, k, v, *_ in cases:   # two calls back to back on one stream
        o, l1, l2 = torch.empty_like(q), torch.empty(q.shape[:3], device=q.device), torch.empty(q.shape[:3], device=q.device)
        desc = sq.make_desc(q, wl.grid, wl.tile, None)
        assert fn(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(o), _p(l1), _p(l2), stream) == 0
        outs.append((o, l1, l2))
    sq.poll_device_error()
    for (wl, q, k, v, ref_o, ref_l1, ref_l2), (o, l1, l2) in zip(cases, outs):
        fp32 = wl.dtype == "f32"
        _close(o, ref_o, fp32, "O")
        assert (l1 - ref_l1).abs().max().item() <= (F32_TOL if fp32 else LSE_TOL)
        assert (l2 - ref_l2).abs().max().item() <= (F32_TOL if fp32 else LSE_TOL)


def test_noalloc_rejects_problems_larger_than_its_scratch(cuda_ok):
    fn = _abi()
    # bf16 [1, 24, 27280, 128]: the local-pass output needs 167.6 MB > 32 MiB
    desc = sq.SquadDesc(1, 24, 128, 31, 22, 40, 1, 11, 20, sq.SQUAD_BF16, 0.0)
    assert 1 * 24 * 27280 * 128 * 2 > SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)   # never touched: the size check comes first
    assert fn(ctypes.byref(desc), fake, fake, fake, fake, None, None, None) == 7   # SQUAD_ERR_WORKSPACE


def test_noalloc_python_binding(cuda_ok):
    wl, inp = _inputs("small_bf16", False)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    ref, *_ = sq.squad_attn_fwd(q, k, v, wl.grid, wl.tile, save=False)
    got = sq.squad_attn_fwd_noalloc(q, k, v, wl.grid, wl.tile)
    sq.poll_device_error()
    _close(got, ref, False, "O")
