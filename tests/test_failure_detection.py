"""Failure detection without a GPU fault.

Every wait in the kernels is bounded by the global timer; a kernel that gives up
sets the library's device error word and returns, and squad_poll_device_error
reports SQUAD_ERR_TIMEOUT. The self-test kernel makes such a wait run out on
purpose (a barrier that nothing completes); the context must stay usable.
"""
import ctypes

import pytest
import torch

import sub_quadratic_two_b200 as sq
from workloads import random_problem

TIMEOUT = 6


def test_selftest_rejects_bad_limits():
    lib = sq.load_library()
    lib.squad_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, ctypes.c_void_p]
    lib.squad_selftest_wait_timeout.restype = ctypes.c_int
    # checked before any CUDA call
    assert lib.squad_selftest_wait_timeout(10, None) == 1
    assert lib.squad_selftest_wait_timeout(100_000_000_000, None) == 1


@pytest.mark.gpu
def test_device_wait_times_out_and_context_survives(cuda_ok):
    sq.poll_device_error()  # clean state
    sq.selftest_wait_timeout(20_000_000)  # 20 ms
    with pytest.raises(sq.SquadError) as e:
        sq.poll_device_error()
    assert e.value.status == TIMEOUT
    sq.poll_device_error()  # the word was cleared
    # the context is still usable: a real call runs and reports no error
    grid, tile = (2, 8, 8), (1, 4, 4)
    inp = random_problem(3, 1, 1, 128, grid, tile, dtype=torch.bfloat16)
    o, *_ = sq.squad_attn_fwd(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), grid, tile)
    sq.poll_device_error()
    assert torch.isfinite(o.float()).all()
