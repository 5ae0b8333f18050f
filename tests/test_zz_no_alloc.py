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


def test_noalloc_matches_the_oracle(cuda_ok):
    # all eight heads of the small bf16 workload against the fp64 oracle directly
    import oracle
    fn = _abi()
    wl, inp = _inputs("small_bf16", False)
    q, k, v = (t.cuda().contiguous() for t in (inp.q, inp.k, inp.v))
    o = torch.empty_like(q)
    l1, l2 = (torch.empty(q.shape[:3], device=q.device) for _ in range(2))
    desc = sq.make_desc(q, wl.grid, wl.tile, None)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert fn(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(o), _p(l1), _p(l2), stream) == 0
    sq.poll_device_error()
    ro, _, rl1, rl2, _ = oracle.squad_fwd(inp.q, inp.k, inp.v, wl.grid, wl.tile)
    _close(o.cpu(), torch.from_numpy(ro), False, "O")
    assert (l1.cpu().double() - torch.from_numpy(rl1)).abs().max().item() <= LSE_TOL
    assert (l2.cpu().double() - torch.from_numpy(rl2)).abs().max().item() <= LSE_TOL


def test_noalloc_at_the_exact_scratch_size(cuda_ok):
    # bf16 [1, 8, 16384, 128]: the local-pass output is exactly 32 MiB, every byte of the
    # scratch array is written and read; compared with squad_attn_fwd (the same kernels,
    # one fused launch) and, on one head, with the oracle
    import oracle
    from workloads import random_problem as rp
    fn = _abi()
    grid, tile = (16, 32, 32), (1, 8, 16)
    inp = rp(99, 1, 8, 128, grid, tile, dtype=torch.bfloat16)
    assert 1 * 8 * 16384 * 128 * 2 == SCRATCH_BYTES
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    o = torch.empty_like(q)
    desc = sq.make_desc(q, grid, tile, None)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        assert fn(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(o), None, None, stream) == 0
    ref, *_ = sq.squad_attn_fwd(q, k, v, grid, tile, save=False)
    sq.poll_device_error()
    _close(o, ref, False, "O vs squad_attn_fwd")
    ro, *_ = oracle.squad_fwd(inp.q[:, 5:6], inp.k[:, 5:6], inp.v[:, 5:6], grid, tile)
    _close(o[:, 5:6].cpu(), torch.from_numpy(ro), False, "O vs oracle")


def test_noalloc_rejects_one_row_past_the_scratch(cuda_ok):
    fn = _abi()
    fake = ctypes.c_void_p(0x10000)   # never touched: the size check comes first
    # fp32 [1, 1, 262144, 32] is exactly 32 MiB: accepted up to the size check; 262145
    # tokens (grid 5 x 13 x 4033) is one 128-byte row more: rejected before any launch
    over = sq.SquadDesc(1, 1, 32, 5, 13, 4033, 1, 1, 1, sq.SQUAD_F32, 0.0)
    assert 262145 * 32 * 4 == SCRATCH_BYTES + 128
    assert fn(ctypes.byref(over), fake, fake, fake, fake, None, None, None) == 7   # SQUAD_ERR_WORKSPACE


def test_noalloc_writes_stay_inside_their_buffers(cuda_ok):
    # guard bands around o, lse1 and lse2 (the only memory the call writes besides its
    # internal scratch): both ends keep their pattern
    from test_guard_bands_gpu import Guarded
    fn = _abi()
    for name in ("small_bf16", "tiny_fp32"):
        wl, inp = _inputs(name, False)
        q, k, v = (t.cuda().contiguous() for t in (inp.q, inp.k, inp.v))
        o = Guarded(q.shape, q.dtype, q.device)
        l1, l2 = (Guarded(q.shape[:3], torch.float32, q.device) for _ in range(2))
        desc = sq.make_desc(q, wl.grid, wl.tile, None)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        assert fn(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(o.t), _p(l1.t), _p(l2.t), stream) == 0
        torch.cuda.synchronize()
        sq.poll_device_error()
        assert o.intact() and l1.intact() and l2.intact(), name
