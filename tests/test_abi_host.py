"""Host-side checks of the C ABI (no GPU needed): exports, argument checks, plans.

Every check here returns before the library makes any CUDA call.
"""
import ctypes
import os
import re

import pytest

import sub_quadratic_two_b200 as sq
from sub_quadratic_two_b200 import SquadDesc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "squad.h")

OK, INVALID, SHAPE, ALIGN, UNSUPPORTED, CUDA, TIMEOUT, WORKSPACE = range(8)


@pytest.fixture(scope="module")
def lib():
    return sq.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(squad_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert "squad_attn_fwd" in names and "squad_attn_bwd" in names
    for name in names:
        assert hasattr(lib, name), name


def test_version_and_strerror(lib):
    assert lib.squad_version() >= 10000
    for code in range(8):
        assert lib.squad_strerror(code)
    assert lib.squad_strerror(99) == b"unknown status"


def _desc(**kw):
    base = dict(B=1, heads=2, d=128, T=4, H=8, W=8, tT=1, tH=4, tW=4, dtype=sq.SQUAD_BF16, scale=0.0)
    base.update(kw)
    return SquadDesc(**base)


FAKE = ctypes.c_void_p(0x10000)        # aligned, never dereferenced: calls fail before any launch
MISALIGNED = ctypes.c_void_p(0x10008)


def _fwd(lib, desc, q=FAKE, k=FAKE, v=FAKE, o=FAKE, o1=FAKE, ws=None, ws_bytes=0):
    return lib.squad_attn_fwd(ctypes.byref(desc), q, k, v, o, o1, None, None, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(tH=3), SHAPE),              # 3 does not divide H=8
    (dict(T=0), SHAPE),
    (dict(tW=-1), SHAPE),
    (dict(dtype=7), INVALID),
    (dict(d=96), UNSUPPORTED),        # bf16 kernels take d in {64, 128}
    (dict(W=256, tW=1), UNSUPPORTED), # a global-pass box row of 256 > 128 tokens
    (dict(dtype=sq.SQUAD_F32, d=48), UNSUPPORTED),
    (dict(B=40000, heads=64, T=32, H=32, W=32, tT=1, tH=1, tW=32), SHAPE),  # rows >= 2^31
])
def test_shape_and_type_errors(lib, kw, code):
    assert _fwd(lib, _desc(**kw)) == code


def test_null_and_alignment_errors(lib):
    d = _desc()
    assert lib.squad_attn_fwd(None, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 0, None) == INVALID
    assert _fwd(lib, d, q=None) == INVALID
    assert _fwd(lib, d, k=MISALIGNED) == ALIGN
    assert _fwd(lib, d, o=MISALIGNED) == ALIGN
    # o1 == NULL needs the workspace
    assert _fwd(lib, d, o1=None) == WORKSPACE
    need = sq.workspace_size(d, 0)
    assert _fwd(lib, d, o1=None, ws=FAKE, ws_bytes=need - 1) == WORKSPACE


def test_backward_argument_errors(lib):
    d = _desc()
    args = [FAKE] * 11
    need = sq.workspace_size(d, 1)
    assert lib.squad_attn_bwd(ctypes.byref(d), *args, FAKE, need - 16, None) == WORKSPACE
    args2 = list(args)
    args2[3] = None  # o
    assert lib.squad_attn_bwd(ctypes.byref(d), *args2, FAKE, need, None) == INVALID
    args3 = list(args)
    args3[8] = MISALIGNED  # dq
    assert lib.squad_attn_bwd(ctypes.byref(d), *args3, FAKE, need, None) == ALIGN


def test_workspace_sizes(lib):
    d = _desc()
    rows = 1 * 2 * 256
    # local-pass output + one progress counter per (batch, head), each part 256-byte aligned
    assert sq.workspace_size(d, 0) == rows * 128 * 2 + 256
    assert sq.workspace_size(d, 2) == 256
    # dO1 (bf16) + dQ2, dK2 (fp32) + two fp32 row vectors, each 256-byte aligned
    assert sq.workspace_size(d, 1) == rows * 128 * 2 + 2 * rows * 128 * 4 + 2 * rows * 4
    with pytest.raises(sq.SquadError):
        sq.workspace_size(d, 5)


def _plan(lib, desc, stage):
    info = (ctypes.c_int * 8)()
    assert lib.squad_plan_info(ctypes.byref(desc), stage, info) == OK
    return list(info)


@pytest.mark.parametrize("grid,tile,expect1,expect2", [
    # local pass of the 5B shape: 220-token windows cut into 120 + 100 token boxes (6 and 5 rows of 20)
    ((31, 22, 40), (1, 11, 20), [220, 124, 2, 120, 20, 6, 1, 2], [124, 220, 1, 124, 2, 2, 31, 1]),
    # long video: 440-token windows -> 4 boxes of 6 rows (online softmax over 2 groups)
    ((61, 22, 40), (1, 22, 20), [440, 122, 4, 120, 20, 6, 1, 2], [122, 440, 1, 122, 2, 1, 61, 1]),
    ((8, 16, 16), (2, 4, 8), [64, 32, 1, 64, 8, 4, 2, 1], [32, 64, 1, 32, 2, 4, 4, 1]),
    ((4, 8, 8), (1, 4, 4), [16, 16, 1, 16, 4, 4, 1, 1], [16, 16, 1, 16, 2, 2, 4, 1]),
])
def test_plans_of_the_workloads(lib, grid, tile, expect1, expect2):
    d = _desc(B=1, heads=24, T=grid[0], H=grid[1], W=grid[2], tT=tile[0], tH=tile[1], tW=tile[2])
    assert _plan(lib, d, 1) == expect1
    assert _plan(lib, d, 2) == expect2


def test_plan_tiles_cover_problem(lib):
    # every tiling covers the problem exactly: nt boxes, the last one ragged
    for grid, tile in [((6, 10, 12), (3, 5, 12)), ((2, 40, 30), (1, 20, 15)), ((9, 4, 4), (1, 2, 2))]:
        d = _desc(T=grid[0], H=grid[1], W=grid[2], tT=tile[0], tH=tile[1], tW=tile[2])
        for stage in (1, 2):
            L, probs, nt, box, a, b, c, kt = _plan(lib, d, stage)
            assert box == a * b * c <= 128
            assert (nt - 1) * box < L <= nt * box


# ---------------------------------------------------------------- more than two passes

def _tiles(*ts):
    flat = [x for t in ts for x in t]
    return len(ts), (ctypes.c_int * len(flat))(*flat)


def _mfwd(lib, desc, tiles, o=FAKE, inter=FAKE, lse=None, ws=None, ws_bytes=0):
    nt, arr = tiles
    return lib.squad_attn_multi_fwd(ctypes.byref(desc), nt, arr, FAKE, FAKE, FAKE, o, inter, lse, ws, ws_bytes, None)


def test_multi_pass_argument_errors(lib):
    d = _desc(T=4, H=8, W=8)
    assert _mfwd(lib, d, _tiles((1, 2, 2), (1, 3, 4))) == SHAPE          # 2 does not divide 3
    assert _mfwd(lib, d, _tiles((1, 4, 4), (1, 2, 2))) == SHAPE          # outer tile smaller than inner
    assert _mfwd(lib, d, _tiles((1, 2, 2), (3, 4, 4))) == SHAPE          # 3 does not divide T=4
    assert _mfwd(lib, d, _tiles(*[(1, 1, 1)] * 5)) == UNSUPPORTED        # at most four tiles
    assert lib.squad_attn_multi_fwd(ctypes.byref(d), 1, None, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 0,
                                    None) == INVALID
    assert _mfwd(lib, d, _tiles((1, 2, 2), (1, 4, 4)), o=MISALIGNED) == ALIGN
    # the one-launch forward's counter workspace: too small, misaligned
    fneed = ctypes.c_size_t(0)
    nt3, arr3 = _tiles((1, 2, 2), (1, 4, 4))
    assert lib.squad_attn_multi_fwd_workspace_size(ctypes.byref(d), nt3, arr3, 1, ctypes.byref(fneed)) == OK
    assert _mfwd(lib, d, (nt3, arr3), ws=FAKE, ws_bytes=fneed.value - 4) == WORKSPACE
    assert _mfwd(lib, d, (nt3, arr3), ws=MISALIGNED, ws_bytes=fneed.value) == ALIGN
    assert lib.squad_attn_multi_fwd_workspace_size(ctypes.byref(d), nt3, arr3, 1, None) == INVALID
    # without inter (inference) the workspace also holds the intermediate outputs
    assert _mfwd(lib, d, (nt3, arr3), inter=None) == WORKSPACE                      # no workspace at all
    assert _mfwd(lib, d, (nt3, arr3), inter=None, ws=FAKE, ws_bytes=fneed.value) == WORKSPACE
    assert lib.squad_attn_multi_fwd_workspace_size(ctypes.byref(d), nt3, arr3, 0, ctypes.byref(fneed)) == OK
    assert _mfwd(lib, d, (nt3, arr3), inter=None, ws=FAKE, ws_bytes=fneed.value - 1) == WORKSPACE
    # bf16: a pass whose box row (t_j / t_{j-1} along W) exceeds 128 tokens
    wide = _desc(T=1, H=1, W=512, tT=1, tH=1, tW=1)
    assert _mfwd(lib, wide, _tiles((1, 1, 2), (1, 1, 512))) == UNSUPPORTED
    nt, arr = _tiles((1, 2, 2), (1, 4, 4))
    need = ctypes.c_size_t(0)
    assert lib.squad_attn_multi_bwd_workspace_size(ctypes.byref(d), nt, arr, ctypes.byref(need)) == OK
    args = [FAKE] * 10  # q, k, v, o, inter, lse, dout, dq, dk, dv
    assert lib.squad_attn_multi_bwd(ctypes.byref(d), nt, arr, *args, FAKE, need.value - 16, None) == WORKSPACE


def test_multi_pass_workspace_size(lib):
    d = _desc(T=4, H=8, W=8)
    nt, arr = _tiles((1, 2, 2), (1, 4, 4))
    got = ctypes.c_size_t(0)
    # forward: one uint32 counter per (pass 2..k, batch, head), rounded up to 256 bytes
    assert lib.squad_attn_multi_fwd_workspace_size(ctypes.byref(d), nt, arr, 1, ctypes.byref(got)) == OK
    assert got.value == 256
    big = _desc(B=3, heads=40, T=4, H=8, W=8)
    assert lib.squad_attn_multi_fwd_workspace_size(ctypes.byref(big), nt, arr, 1, ctypes.byref(got)) == OK
    assert got.value == 1024                     # passes 2 and 3 x 120 heads x 4 bytes = 960, rounded up
    # inference: the outputs of passes 1 and 2 (bf16 [3, 40, 256, 128]) before the counters
    assert lib.squad_attn_multi_fwd_workspace_size(ctypes.byref(big), nt, arr, 0, ctypes.byref(got)) == OK
    assert got.value == 2 * 3 * 40 * 256 * 128 * 2 + 1024

    assert lib.squad_attn_multi_bwd_workspace_size(ctypes.byref(d), nt, arr, ctypes.byref(got)) == OK
    rows = 1 * 2 * 256
    # two bf16 upstream gradients, four fp32 accumulators, three fp32 row vectors
    assert got.value == 2 * rows * 128 * 2 + 4 * rows * 128 * 4 + 3 * rows * 4


# ---------------------------------------------------------------- forward from host memory

def test_host_forward_workspace_and_argument_errors(lib):
    d = _desc(B=2, heads=3, T=4, H=8, W=8)          # 6 slices of 256 tokens, bf16, d = 128
    got = ctypes.c_size_t(0)
    assert lib.squad_attn_fwd_host_workspace_size(ctypes.byref(d), 4, ctypes.byref(got)) == OK
    chunk = 4 * 256 * 128 * 2
    fwd = ctypes.c_size_t(0)
    dc = _desc(B=1, heads=4, T=4, H=8, W=8)
    assert lib.squad_attn_workspace_size(ctypes.byref(dc), 0, ctypes.byref(fwd)) == OK
    assert got.value == 2 * 4 * chunk + fwd.value     # two sets of q, k, v, o chunks + the chunk forward's
    assert lib.squad_attn_fwd_host_workspace_size(ctypes.byref(d), 0, ctypes.byref(got)) == INVALID
    assert lib.squad_attn_fwd_host_workspace_size(ctypes.byref(d), 4, None) == INVALID
    big = ctypes.c_size_t(0)
    assert lib.squad_attn_fwd_host_workspace_size(ctypes.byref(d), 100, ctypes.byref(big)) == OK  # capped at 6
    need = ctypes.c_size_t(0)
    assert lib.squad_attn_fwd_host_workspace_size(ctypes.byref(d), 4, ctypes.byref(need)) == OK
    S1, S2, S3 = ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000), ctypes.c_void_p(0x40000)
    def call(ws=FAKE, nb=None, s=(S1, S2, S3), q=FAKE, chunk=4):
        return lib.squad_attn_fwd_host(ctypes.byref(d), q, FAKE, FAKE, FAKE, chunk, ws,
                                       need.value if nb is None else nb, *s)
    assert call(q=None) == INVALID
    assert call(chunk=0) == INVALID
    assert call(s=(S1, S2, S2)) == INVALID            # the three streams must differ
    assert call(s=(S1, S1, S3)) == INVALID
    assert call(s=(S1, None, S3)) == INVALID
    assert call(ws=MISALIGNED) == ALIGN
    assert call(ws=None) == WORKSPACE
    assert call(nb=need.value - 16) == WORKSPACE
