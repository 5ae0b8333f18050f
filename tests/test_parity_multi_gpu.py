"""GPU parity of the k-pass entry points (passes over nested tiles) against the oracle.

fp32: max |err| <= 1e-5, as for the two-pass operator. bf16: the two-pass
tolerances (forward max 1.5e-2, mean 2e-3; gradients max 3e-2) budget two
passes, each of which rounds its probabilities to bf16 before the P.V product and
stores its output in bf16; a pass passes the error of its values on through a
convex combination, so the errors of k passes add. The bf16 bounds here are
therefore the two-pass ones times k / 2 (three passes: max 2.25e-2, mean 3e-3;
gradients 4.5e-2). tests/test_kpass_error_budget.py pins this budget on the CPU with a
model of the two roundings per pass (additivity over passes; three passes on the
27,280-token shape reach about 2e-2 from rounding alone). Reading of the
pages' outlook on composing more than two passes ("SQuad: Sub-Quadratic
Attention Distillation for Efficient Video Generation", gist.science technical
summary, Significance and Claims): nested tiles, pass j attends within a
t_j-window among tokens at the same position in their t_{j-1}-window.
"""
import numpy as np
import pytest
import torch

import oracle
import sub_quadratic_two_b200 as sq
from workloads import WORKLOADS, make_inputs, random_problem

pytestmark = pytest.mark.gpu

F32_TOL = 1e-5
BF16_MAX, BF16_MEAN, GRAD_MAX = 1.5e-2, 2e-3, 3e-2   # two passes


def _bf16_tol(npasses):
    """(forward max, forward mean, gradient max) for npasses bf16 passes."""
    f = npasses / 2.0
    return BF16_MAX * f, BF16_MEAN * f, GRAD_MAX * f


def _np(t):
    return t.detach().cpu().double().numpy()


def _err(a, b):
    e = np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))
    return float(e.max()), float(e.mean())


def _err_scaled(a, b):
    """max |a - b| / max(1, |b|): the gradient bound at large magnitudes, where the bf16
    rounding of the result is relative (tests/test_kpass_error_budget.py)."""
    b = np.asarray(b, np.float64)
    return float((np.abs(np.asarray(a, np.float64) - b) / np.maximum(1.0, np.abs(b))).max())


def _gpu_fwd_bwd(inp, grid, tiles, scale=None):
    q, k, v, do = (t.contiguous().cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    o, inter, lse = sq.squad_attn_multi_fwd(q, k, v, grid, tiles, scale)
    grads = sq.squad_attn_multi_bwd(q, k, v, o, inter, lse, do, grid, tiles, scale)
    sq.poll_device_error()
    return o, inter, lse, grads


@pytest.mark.parametrize("grid,tiles,d", [
    ((2, 4, 8), [(1, 2, 2), (2, 2, 4)], 64),
    ((2, 4, 8), [(1, 1, 2), (1, 2, 2), (2, 2, 4)], 32),   # four passes
    ((3, 6, 4), [(1, 3, 1), (3, 3, 2)], 96),
])
def test_fp32_passes_forward_and_backward(cuda_ok, grid, tiles, d):
    inp = random_problem(51, 2, 2, d, grid, (1, 1, 1), dtype=torch.float32, with_do=True)
    o, inter, lse, grads = _gpu_fwd_bwd(inp, grid, tiles)
    ro, rinter, rlse, _ = oracle.squad_fwd_multi(inp.q, inp.k, inp.v, grid, tiles)
    assert _err(_np(o), ro)[0] <= F32_TOL
    assert _err(_np(inter), rinter)[0] <= F32_TOL
    assert _err(_np(lse), rlse)[0] <= F32_TOL
    ref = oracle.squad_bwd_multi(inp.q, inp.k, inp.v, inp.do, grid, tiles)
    for name, a, b in zip(("dQ", "dK", "dV"), grads, ref):
        assert _err(_np(a), b)[0] <= F32_TOL, name


@pytest.mark.parametrize("grid,tiles,d", [
    ((4, 22, 40), [(1, 1, 20), (1, 11, 20)], 128),     # 20 | 11 | 16 tokens per group
    ((2, 44, 40), [(1, 2, 20), (1, 22, 20)], 128),     # 40-token, 11-token, 8-token groups
    ((80, 8, 8), [(1, 2, 2), (2, 4, 4)], 128),         # last pass: 160-token groups in two boxes
    ((4, 16, 16), [(1, 4, 4), (2, 8, 8)], 64),         # d = 64
    ((2, 8, 16), [(1, 1, 2), (1, 2, 4), (2, 4, 8)], 128),  # four passes
    # small problems packed several to a box, along each box dimension, ragged last groups:
    ((4, 22, 40), [(1, 1, 20), (2, 11, 20)], 128),     # pass 2: 22-token groups packed along a (5 per box)
    ((4, 22, 40), [(2, 1, 20), (2, 11, 20)], 128),     # pass 1: 40-token windows packed along b (3 per box, 22 = 7 x 3 + 1)
])
def test_bf16_passes_forward_and_backward(cuda_ok, grid, tiles, d):
    inp = random_problem(53, 1, 2, d, grid, (1, 1, 1), dtype=torch.bfloat16, k_bias_std=1.0, with_do=True)
    o, inter, lse, grads = _gpu_fwd_bwd(inp, grid, tiles)
    ro, rinter, rlse, _ = oracle.squad_fwd_multi(inp.q, inp.k, inp.v, grid, tiles)
    fmax, fmean, gmax = _bf16_tol(len(tiles) + 1)
    mx, mean = _err(_np(o), ro)
    assert mx <= fmax and mean <= fmean, (mx, mean)
    for j in range(len(tiles)):
        # the output of pass j + 1 carries the rounding of j + 1 passes
        jmax, jmean, _ = _bf16_tol(max(2, j + 1))
        mx, mean = _err(_np(inter[j]), rinter[j])
        assert mx <= jmax and mean <= jmean, (j, mx, mean)
    ref = oracle.squad_bwd_multi(inp.q, inp.k, inp.v, inp.do, grid, tiles)
    for name, a, b in zip(("dQ", "dK", "dV"), grads, ref):
        assert np.isfinite(_np(a)).all(), name
        assert _err(_np(a), b)[0] <= gmax, name


def test_one_tile_matches_the_two_pass_operator(cuda_ok):
    # 220-token windows and 80-token groups: neither pass is packed, so the k-pass
    # forward runs exactly the two-pass operator's boxes
    grid, tile = (20, 22, 40), (1, 11, 20)
    inp = random_problem(55, 1, 2, 128, grid, tile, dtype=torch.bfloat16, with_do=True)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    o, inter, lse = sq.squad_attn_multi_fwd(q, k, v, grid, [tile])
    o2, o1, l1, l2 = sq.squad_attn_fwd(q, k, v, grid, tile)
    sq.poll_device_error()
    assert torch.equal(o, o2) and torch.equal(inter[0], o1)
    assert torch.equal(lse[0], l1) and torch.equal(lse[1], l2)


def test_one_tile_packed_global_pass(cuda_ok):
    # 16-token groups: the k-pass forward packs eight of them into a box (the two-pass
    # operator does not), so both are compared with the oracle
    grid, tile = (4, 22, 40), (1, 11, 20)
    inp = random_problem(56, 1, 2, 128, grid, tile, dtype=torch.bfloat16, with_do=True)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    o, inter, lse = sq.squad_attn_multi_fwd(q, k, v, grid, [tile])
    o2, o1, l1, l2 = sq.squad_attn_fwd(q, k, v, grid, tile)
    sq.poll_device_error()
    ro, ro1, rl1, rl2, _ = oracle.squad_fwd(inp.q, inp.k, inp.v, grid, tile)
    for a in (o, o2):
        mx, mean = _err(_np(a), ro)
        assert mx <= BF16_MAX and mean <= BF16_MEAN, (mx, mean)
    assert torch.equal(inter[0], o1)  # the local pass (220-token windows) is not packed
    assert _err(_np(lse[1]), rl2)[0] <= 2e-3
    assert _err(_np(l2), rl2)[0] <= 2e-3


def test_autograd_through_three_passes(cuda_ok):
    grid, tiles = (2, 8, 8), [(1, 2, 2), (2, 4, 4)]
    inp = random_problem(57, 1, 2, 128, grid, (1, 1, 1), dtype=torch.bfloat16, with_do=True)
    q, k, v = (t.cuda().requires_grad_(True) for t in (inp.q, inp.k, inp.v))
    o = sq.attention_multi(q, k, v, grid, tiles)
    o.backward(inp.do.cuda())
    ref = oracle.squad_bwd_multi(inp.q, inp.k, inp.v, inp.do, grid, tiles)
    gmax = _bf16_tol(len(tiles) + 1)[2]
    for name, t, r in zip(("dQ", "dK", "dV"), (q, k, v), ref):
        assert _err(_np(t.grad), r)[0] <= gmax, name


def test_three_passes_on_the_video_shape(cuda_ok):
    # the 27,280-token shape with windows of 220 = 20 x 11: groups of 20, 11 and 124 tokens
    wl = WORKLOADS["wan5b_fwd"]
    inp = make_inputs(wl)
    tiles = [(1, 1, 20), (1, 11, 20)]
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    o, _, _ = sq.squad_attn_multi_fwd(q, k, v, wl.grid, tiles)
    sq.poll_device_error()
    fmax, fmean, _ = _bf16_tol(3)
    for h in (0, 17):
        sel = (slice(0, 1), slice(h, h + 1))
        ro, _, _, _ = oracle.squad_fwd_multi(inp.q[sel], inp.k[sel], inp.v[sel], wl.grid, tiles)
        mx, mean = _err(_np(o[sel]), ro)
        assert mx <= fmax and mean <= fmean, (h, mx, mean)


def test_packed_passes_are_deterministic(cuda_ok):
    # packed boxes (20-token windows six to a box along c, then 22-token groups five to a
    # box along a) run the same MMAs in the same order on every call: bitwise repeatable
    grid, tiles = (4, 22, 40), [(1, 1, 20), (2, 11, 20)]
    inp = random_problem(59, 1, 2, 128, grid, (1, 1, 1), dtype=torch.bfloat16)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    first = sq.squad_attn_multi_fwd(q, k, v, grid, tiles)
    second = sq.squad_attn_multi_fwd(q, k, v, grid, tiles)
    sq.poll_device_error()
    for a, b in zip(first, second):
        assert torch.equal(a, b)


@pytest.mark.parametrize("B,heads,grid,tiles,d", [
    (1, 1, (2, 8, 16), [(1, 1, 2), (1, 2, 4), (2, 4, 8)], 128),   # one head: no full block
    (1, 3, (4, 22, 40), [(1, 1, 20), (2, 11, 20)], 128),          # packed passes, heads < 2 lags
    (2, 3, (2, 8, 16), [(1, 2, 2), (1, 4, 4)], 64),
    (1, 7, (2, 8, 16), [(1, 1, 2), (1, 2, 2), (1, 4, 8), (2, 8, 8)], 64),   # five passes
    (2, 5, (2, 16, 64), [(1, 4, 64), (2, 8, 64)], 128),           # 256-token problems: two boxes each
])
def test_one_launch_equals_one_launch_per_pass(cuda_ok, B, heads, grid, tiles, d):
    # the chained launch runs each job exactly as the per-pass launches do: bitwise equal
    inp = random_problem(61, B, heads, d, grid, (1, 1, 1), dtype=torch.bfloat16)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    one = sq.squad_attn_multi_fwd(q, k, v, grid, tiles, one_launch=True)
    per = sq.squad_attn_multi_fwd(q, k, v, grid, tiles, one_launch=False)
    inf, _, _ = sq.squad_attn_multi_fwd(q, k, v, grid, tiles, save=False)   # intermediates in scratch
    sq.poll_device_error()
    for name, a, b in zip(("o", "inter", "lse"), one, per):
        assert torch.equal(a, b), name
    assert torch.equal(inf, one[0])


def test_one_launch_three_passes_full_size(cuda_ok):
    # the 27,280-token shape, 24 heads, three passes in one launch: bitwise the per-pass result,
    # and within the three-pass bf16 budget of the oracle on two heads
    wl = WORKLOADS["wan5b_fwd"]
    inp = make_inputs(wl)
    tiles = [(1, 1, 20), (1, 11, 20)]
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    one = sq.squad_attn_multi_fwd(q, k, v, wl.grid, tiles, one_launch=True)
    per = sq.squad_attn_multi_fwd(q, k, v, wl.grid, tiles, one_launch=False)
    inf, _, _ = sq.squad_attn_multi_fwd(q, k, v, wl.grid, tiles, save=False)
    sq.poll_device_error()
    for name, a, b in zip(("o", "inter", "lse"), one, per):
        assert torch.equal(a, b), name
    assert torch.equal(inf, one[0])
    fmax, fmean, _ = _bf16_tol(3)
    for h in (5, 23):
        sel = (slice(0, 1), slice(h, h + 1))
        ro, _, _, _ = oracle.squad_fwd_multi(inp.q[sel], inp.k[sel], inp.v[sel], wl.grid, tiles)
        mx, mean = _err(_np(one[0][sel]), ro)
        assert mx <= fmax and mean <= fmean, (h, mx, mean)


def test_three_passes_backward_full_size(cuda_ok):
    # the 27,280-token shape, 24 heads, three passes: forward in one launch, backward with the
    # 20- and 11-token groups packed six and ten to a box; two heads against the oracle
    # (head 20 has gradients up to 8.8: the bound applies to |err| / max(1, |ref|))
    wl = WORKLOADS["wan5b_fwd"]
    inp = make_inputs(wl)
    tiles = [(1, 1, 20), (1, 11, 20)]
    g = torch.Generator().manual_seed(97)
    do = torch.randn(inp.q.shape, generator=g).to(torch.bfloat16)
    q, k, v, dog = (t.cuda() for t in (inp.q, inp.k, inp.v, do))
    o, inter, lse = sq.squad_attn_multi_fwd(q, k, v, wl.grid, tiles)
    dq, dk, dv = sq.squad_attn_multi_bwd(q, k, v, o, inter, lse, dog, wl.grid, tiles)
    sq.poll_device_error()
    _, _, gmax = _bf16_tol(3)
    for h in (3, 20):
        sel = (slice(0, 1), slice(h, h + 1))
        ref = oracle.squad_bwd_multi(inp.q[sel], inp.k[sel], inp.v[sel], do[sel], wl.grid, tiles)
        for name, a, b in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref):
            assert np.isfinite(_np(a[sel])).all(), name
            assert _err_scaled(_np(a[sel]), b) <= gmax, (h, name)


@pytest.mark.parametrize("d", [64, 128])
def test_packed_passes_batch_two_forward_and_backward(cuda_ok, d):
    # B = 2 with packed boxes in both directions (20-token windows six to a box, 22-token
    # groups five to a box): every (batch, head) slice against the oracle
    grid, tiles = (4, 22, 40), [(1, 1, 20), (2, 11, 20)]
    inp = random_problem(87, 2, 2, d, grid, (1, 1, 1), dtype=torch.bfloat16, with_do=True)
    o, inter, lse, grads = _gpu_fwd_bwd(inp, grid, tiles)
    ro, _, _, _ = oracle.squad_fwd_multi(inp.q, inp.k, inp.v, grid, tiles)
    fmax, fmean, gmax = _bf16_tol(3)
    mx, mean = _err(_np(o), ro)
    assert mx <= fmax and mean <= fmean, (mx, mean)
    ref = oracle.squad_bwd_multi(inp.q, inp.k, inp.v, inp.do, grid, tiles)
    for name, a, b in zip(("dQ", "dK", "dV"), grads, ref):
        assert np.isfinite(_np(a)).all(), name
        assert _err(_np(a), b)[0] <= gmax, name
