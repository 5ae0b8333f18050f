"""The Python binding refuses tensors whose extent the C ABI would have to trust.

The C entry points take plain pointers and derive every extent from the
descriptor, so a saved LSE or intermediate of the wrong shape, dtype or device
(or a caller-provided output of the wrong shape) would make a kernel read or
write outside it. The binding checks them before any call; nothing here
launches a kernel with a bad tensor.
"""
import pytest
import torch

import sub_quadratic_two_b200 as sq
from workloads import WORKLOADS, make_inputs, random_problem

pytestmark = pytest.mark.gpu


def test_backward_rejects_mismatched_saved_tensors(cuda_ok):
    grid, tile = (2, 8, 8), (1, 4, 4)
    inp = random_problem(61, 1, 2, 64, grid, tile, dtype=torch.bfloat16, with_do=True)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    o, o1, l1, l2 = sq.squad_attn_fwd(q, k, v, grid, tile)
    with pytest.raises(ValueError):
        sq.squad_attn_bwd(q, k, v, o, o1, l1.to(torch.bfloat16), l2, do, grid, tile)
    with pytest.raises(ValueError):
        sq.squad_attn_bwd(q, k, v, o, o1, l1, l2[:, :1].contiguous(), do, grid, tile)
    with pytest.raises(ValueError):
        sq.squad_attn_bwd(q, k, v, o, o1, l1.cpu(), l2, do, grid, tile)
    o2, inter, lse = sq.squad_attn_multi_fwd(q, k, v, grid, [tile])
    with pytest.raises(ValueError):
        sq.squad_attn_multi_bwd(q, k, v, o2, inter[:, :, :1].contiguous(), lse, do, grid, [tile])
    with pytest.raises(ValueError):
        sq.squad_attn_multi_bwd(q, k, v, o2, inter, lse.double(), do, grid, [tile])
    sq.poll_device_error()


def test_forward_rejects_mismatched_outputs(cuda_ok):
    grid, tile = (2, 8, 8), (1, 4, 4)
    inp = random_problem(62, 1, 2, 64, grid, tile, dtype=torch.bfloat16)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    with pytest.raises(ValueError):
        sq.squad_attn_fwd(q, k, v, grid, tile, out=torch.empty(5, device=q.device, dtype=q.dtype))
    with pytest.raises(ValueError):
        sq.squad_attn_fwd(q, k, v, grid, tile, out=torch.empty_like(q, dtype=torch.float32))
    with pytest.raises(ValueError):
        sq.squad_attn_fwd_pass(1, q, k, v, torch.empty_like(q), grid, tile,
                               lse=torch.empty(q.shape[:2], device=q.device, dtype=torch.float32))
    with pytest.raises(ValueError):
        sq.squad_attn_fwd_noalloc(q, k, v, grid, tile, lse1=torch.empty(3, device=q.device, dtype=torch.float32))
    sq.poll_device_error()


def test_repeated_call_reuses_its_tensor_maps(cuda_ok):
    # a forward launch needs eight TMA tensor maps; a second call with the same pointers
    # and shapes takes all eight from the library's cache and encodes none
    wl = WORKLOADS["small_bf16"]
    inp = make_inputs(wl)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    o = torch.empty_like(q)
    ws = torch.empty(sq.workspace_size(sq.make_desc(q, wl.grid, wl.tile, None), 0), device="cuda", dtype=torch.uint8)
    sq.squad_attn_fwd(q, k, v, wl.grid, wl.tile, save=False, out=o, workspace=ws)
    hits0, misses0 = sq.tmap_cache_stats()
    sq.squad_attn_fwd(q, k, v, wl.grid, wl.tile, save=False, out=o, workspace=ws)
    hits1, misses1 = sq.tmap_cache_stats()
    sq.poll_device_error()
    assert misses1 == misses0 and hits1 == hits0 + 8
    o2 = torch.empty_like(q)   # another output buffer: only its map is new
    sq.squad_attn_fwd(q, k, v, wl.grid, wl.tile, save=False, out=o2, workspace=ws)
    hits2, misses2 = sq.tmap_cache_stats()
    sq.poll_device_error()
    assert misses2 == misses1 + 1 and hits2 == hits1 + 7
    assert torch.equal(o, o2)


@pytest.mark.parametrize("name,chunk", [("wan5b_fwd", 4), ("wan5b_fwd", 5), ("wan5b_fwd", 24),
                                        ("small_bf16", 3), ("tiny_fp32", 1)])
def test_forward_from_host_memory_equals_the_device_forward(cuda_ok, name, chunk):
    # chunks of (batch, head) slices copied in, computed and copied out on three streams:
    # the same kernels on the same problems, so bitwise the device call's result
    from workloads import WORKLOADS, make_inputs
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    hq, hk, hv = (t.contiguous().pin_memory() for t in (inp.q, inp.k, inp.v))
    out = sq.attention_host(hq, hk, hv, wl.grid, wl.tile, slices_per_chunk=chunk)
    sq.poll_device_error()
    ref = sq.attention(*(t.cuda() for t in (inp.q, inp.k, inp.v)), wl.grid, wl.tile).cpu()
    assert not out.is_cuda
    assert torch.equal(out, ref)


def test_forward_from_pageable_host_memory(cuda_ok):
    # pageable inputs and output: the copies serialise but the result is the same
    from workloads import WORKLOADS, make_inputs
    wl = WORKLOADS["small_bf16"]
    inp = make_inputs(wl)
    out = torch.empty(inp.q.shape, dtype=inp.q.dtype)
    sq.attention_host(inp.q.contiguous(), inp.k.contiguous(), inp.v.contiguous(), wl.grid, wl.tile, out=out,
                      slices_per_chunk=2)
    ref = sq.attention(*(t.cuda() for t in (inp.q, inp.k, inp.v)), wl.grid, wl.tile).cpu()
    assert torch.equal(out, ref)


def test_forward_from_host_memory_batch_and_d64(cuda_ok):
    # B = 2, 3 heads (6 slices in chunks of 4: one full, one ragged), d = 64
    grid, tile = (4, 8, 8), (1, 4, 4)
    inp = random_problem(83, 2, 3, 64, grid, tile, dtype=torch.bfloat16)
    hq, hk, hv = (t.contiguous().pin_memory() for t in (inp.q, inp.k, inp.v))
    out = sq.attention_host(hq, hk, hv, grid, tile, slices_per_chunk=4)
    ref = sq.attention(*(t.cuda() for t in (inp.q, inp.k, inp.v)), grid, tile).cpu()
    assert torch.equal(out, ref)
