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
from workloads import random_problem

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
