"""Guard bands around every buffer the library writes (a bounds check without a sanitizer).

Each output, saved statistic, intermediate and workspace is the middle of a larger
allocation whose two ends hold a fixed bit pattern. The entry points are called
through the C ABI with exactly the documented extents; afterwards both ends must
still hold the pattern, so a kernel that wrote outside its buffer (a wrong row
index, a ragged tile, a packed group past its digit, a workspace overrun) fails here
instead of corrupting a neighbour. Only in-bounds accesses are made: the guards are
part of the allocation.
"""
import ctypes
import math

import pytest
import torch

import sub_quadratic_two_b200 as sq
from workloads import random_problem

pytestmark = pytest.mark.gpu

GUARD_BYTES = 16 << 10
PATTERN = {1: 0x5A, 2: 0x7ABC, 4: 0x7ABCDEF0}


class Guarded:
    """A tensor of `shape` and `dtype` with GUARD_BYTES of fixed pattern on each side."""

    def __init__(self, shape, dtype, device):
        self.shape = tuple(shape)
        esz = torch.empty((), dtype=dtype).element_size()
        self.g = GUARD_BYTES // esz
        n = math.prod(self.shape)
        self.buf = torch.empty(n + 2 * self.g, dtype=dtype, device=device)
        self.ints = self.buf.view({1: torch.uint8, 2: torch.int16, 4: torch.int32}[esz])
        self.pattern = PATTERN[esz]
        self.ints.fill_(self.pattern)
        self.t = self.buf[self.g:self.g + n].view(self.shape)

    def intact(self):
        return bool((self.ints[:self.g] == self.pattern).all()) and bool((self.ints[-self.g:] == self.pattern).all())


def _p(x):
    return ctypes.c_void_p(x.t.data_ptr() if isinstance(x, Guarded) else x.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _two_pass_case(grid, tile, heads, d, dtype, seed):
    lib = sq.load_library()
    inp = random_problem(seed, 1, heads, d, grid, tile, dtype=dtype, with_do=True)
    dev = torch.device("cuda", 0)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    desc = sq.make_desc(q, grid, tile, None)
    rows = q.shape[:3]
    outs = {n: Guarded(q.shape, q.dtype, dev) for n in ("o", "o1", "dq", "dk", "dv")}
    outs.update({n: Guarded(rows, torch.float32, dev) for n in ("lse1", "lse2")})
    fws, bws = sq.workspace_size(desc, 2), sq.workspace_size(desc, 1)
    outs["fws"] = Guarded((fws,), torch.uint8, dev)
    outs["bws"] = Guarded((bws,), torch.uint8, dev)
    assert lib.squad_attn_fwd(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(outs["o"]), _p(outs["o1"]),
                              _p(outs["lse1"]), _p(outs["lse2"]), _p(outs["fws"]), fws, _stream()) == 0
    assert lib.squad_attn_bwd(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(outs["o"]), _p(outs["o1"]),
                              _p(outs["lse1"]), _p(outs["lse2"]), _p(do), _p(outs["dq"]), _p(outs["dk"]),
                              _p(outs["dv"]), _p(outs["bws"]), bws, _stream()) == 0
    torch.cuda.synchronize()
    sq.poll_device_error()
    return outs


@pytest.mark.parametrize("grid,tile,heads,d,dtype", [
    ((4, 22, 40), (1, 11, 20), 2, 128, torch.bfloat16),   # 220-token windows: ragged boxes 120 + 100
    ((8, 16, 16), (2, 4, 8), 3, 64, torch.bfloat16),      # d = 64, tT > 1
    ((2, 10, 88), (1, 5, 88), 1, 128, torch.bfloat16),    # 440-token windows: five 88-row boxes, online softmax
    ((4, 8, 8), (1, 4, 4), 2, 64, torch.float32),         # fp32 path
])
def test_two_pass_writes_stay_inside_their_buffers(cuda_ok, grid, tile, heads, d, dtype):
    outs = _two_pass_case(grid, tile, heads, d, dtype, 71)
    for name, g in outs.items():
        assert g.intact(), name


@pytest.mark.parametrize("grid,tiles,dtype", [
    ((4, 22, 40), [(1, 1, 20), (2, 11, 20)], torch.bfloat16),   # packed along c, then along a
    ((4, 22, 40), [(2, 1, 20), (2, 11, 20)], torch.bfloat16),   # packed along b, ragged last group
    ((2, 8, 16), [(1, 1, 2), (1, 2, 4), (2, 4, 8)], torch.bfloat16),
    ((2, 4, 8), [(1, 2, 2), (2, 2, 4)], torch.float32),
])
def test_k_pass_writes_stay_inside_their_buffers(cuda_ok, grid, tiles, dtype):
    lib = sq.load_library()
    inp = random_problem(73, 1, 2, 128 if dtype == torch.bfloat16 else 64, grid, (1, 1, 1), dtype=dtype,
                         with_do=True)
    dev = torch.device("cuda", 0)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    desc = sq.make_desc(q, grid, tiles[0], None)
    nt = len(tiles)
    tarr = (ctypes.c_int * (3 * nt))(*[x for t in tiles for x in t])
    o = Guarded(q.shape, q.dtype, dev)
    inter = Guarded((nt,) + tuple(q.shape), q.dtype, dev)
    lse = Guarded((nt + 1,) + tuple(q.shape[:3]), torch.float32, dev)
    dq, dk, dv = (Guarded(q.shape, q.dtype, dev) for _ in range(3))
    need = ctypes.c_size_t(0)
    assert lib.squad_attn_multi_bwd_workspace_size(ctypes.byref(desc), nt, tarr, ctypes.byref(need)) == 0
    ws = Guarded((need.value,), torch.uint8, dev)
    fneed = ctypes.c_size_t(0)
    assert lib.squad_attn_multi_fwd_workspace_size(ctypes.byref(desc), nt, tarr, 1, ctypes.byref(fneed)) == 0
    fws = Guarded((fneed.value,), torch.uint8, dev)
    assert lib.squad_attn_multi_fwd(ctypes.byref(desc), nt, tarr, _p(q), _p(k), _p(v), _p(o), _p(inter), _p(lse),
                                    _p(fws), fneed.value, _stream()) == 0
    assert lib.squad_attn_multi_bwd(ctypes.byref(desc), nt, tarr, _p(q), _p(k), _p(v), _p(o), _p(inter), _p(lse),
                                    _p(do), _p(dq), _p(dk), _p(dv), _p(ws), need.value, _stream()) == 0
    torch.cuda.synchronize()
    sq.poll_device_error()
    for name, g in (("o", o), ("inter", inter), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv), ("ws", ws),
                    ("fws", fws)):
        assert g.intact(), name


@pytest.mark.parametrize("grid,tile,heads,d", [
    ((4, 22, 40), (1, 11, 20), 2, 128),   # 220-token windows: ragged boxes 120 + 100
    ((2, 10, 88), (1, 5, 88), 1, 128),    # 440-token windows in five boxes
    ((8, 16, 16), (2, 4, 8), 3, 64),      # d = 64, tT > 1
])
def test_inference_forward_writes_stay_inside_their_buffers(cuda_ok, grid, tile, heads, d):
    # o1 == NULL: the local-pass output and the per-head counters live in the workspace
    # (squad_attn_workspace_size(desc, 0)), and consumed local-pass rows are dropped from
    # L2 after the global pass reads them
    lib = sq.load_library()
    inp = random_problem(75, 1, heads, d, grid, tile, dtype=torch.bfloat16)
    dev = torch.device("cuda", 0)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    desc = sq.make_desc(q, grid, tile, None)
    o = Guarded(q.shape, q.dtype, dev)
    need = sq.workspace_size(desc, 0)
    ws = Guarded((need,), torch.uint8, dev)
    assert lib.squad_attn_fwd(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(o), None, None, None, _p(ws), need,
                              _stream()) == 0
    torch.cuda.synchronize()
    sq.poll_device_error()
    assert o.intact() and ws.intact()
    ref, *_ = sq.squad_attn_fwd(q, k, v, grid, tile, save=True)
    sq.poll_device_error()
    assert torch.equal(o.t, ref)


@pytest.mark.parametrize("grid,tiles,dtype", [
    ((4, 22, 40), [(1, 1, 20), (2, 11, 20)], torch.bfloat16),
    ((2, 4, 8), [(1, 2, 2), (2, 2, 4)], torch.float32),
])
def test_k_pass_inference_writes_stay_inside_their_buffers(cuda_ok, grid, tiles, dtype):
    # no inter: the intermediate outputs live in the workspace (and leave L2 unwritten on bf16)
    lib = sq.load_library()
    inp = random_problem(79, 1, 3, 128 if dtype == torch.bfloat16 else 64, grid, (1, 1, 1), dtype=dtype)
    dev = torch.device("cuda", 0)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    desc = sq.make_desc(q, grid, tiles[0], None)
    nt = len(tiles)
    tarr = (ctypes.c_int * (3 * nt))(*[x for t in tiles for x in t])
    o = Guarded(q.shape, q.dtype, dev)
    need = ctypes.c_size_t(0)
    assert lib.squad_attn_multi_fwd_workspace_size(ctypes.byref(desc), nt, tarr, 0, ctypes.byref(need)) == 0
    ws = Guarded((need.value,), torch.uint8, dev)
    assert lib.squad_attn_multi_fwd(ctypes.byref(desc), nt, tarr, _p(q), _p(k), _p(v), _p(o), None, None,
                                    _p(ws), need.value, _stream()) == 0
    torch.cuda.synchronize()
    sq.poll_device_error()
    assert o.intact() and ws.intact()
    ref, _, _ = sq.squad_attn_multi_fwd(q, k, v, grid, tiles)
    assert torch.equal(o.t, ref)
