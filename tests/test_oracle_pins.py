"""Pins for the fp64 oracle: facts that do not come from the oracle itself.

Each check is chosen so that a plausible slip in the oracle (a wrong window or
group index, a dropped max-subtraction, V used where the local output belongs,
a wrong scale, a sign or transpose in the gradient) fails at least one of them.
Operator definition: "SQuad: Sub-Quadratic Attention Distillation for Efficient
Video Generation", gist.science technical summary, Methodology section 1.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from workloads import random_problem

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _coords(grid):
    T, H, W = grid
    t, y, x = np.unravel_index(np.arange(T * H * W), (T, H, W))  # x fastest
    return t, y, x


def _block_masks(grid, tile):
    """Boolean masks from the geometric definition: same window / same in-window position."""
    t, y, x = _coords(grid)
    tT, tH, tW = tile
    win = np.stack([t // tT, y // tH, x // tW], 1)
    pos = np.stack([t % tT, y % tH, x % tW], 1)
    m1 = (win[:, None, :] == win[None, :, :]).all(-1)
    m2 = (pos[:, None, :] == pos[None, :, :]).all(-1)
    return torch.from_numpy(m1), torch.from_numpy(m2)


def _masked_sdpa_two_pass(q, k, v, grid, tile, scale=None):
    """Both passes as library SDPA calls with block masks (float64, CPU)."""
    m1, m2 = _block_masks(grid, tile)
    o1 = F.scaled_dot_product_attention(q, k, v, attn_mask=m1, scale=scale)
    o = F.scaled_dot_product_attention(q, k, o1, attn_mask=m2, scale=scale)
    return o, o1


def _f64(x):
    return x.double()


# ---------------------------------------------------------------- hand-derived case

def test_golden_two_window_closed_form():
    g = json.load(open(os.path.join(GOLDEN, "two_window_closed_form.json")))
    q = np.array(g["q"]).reshape(1, 1, 4, 1)
    k = np.array(g["k"]).reshape(1, 1, 4, 1)
    v = np.array(g["v"]).reshape(1, 1, 4, 1)
    o, o1, l1, l2, _ = oracle.squad_fwd(q, k, v, tuple(g["grid"]), tuple(g["tile"]), scale=g["scale"])
    np.testing.assert_allclose(o1.ravel(), g["o1"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(o.ravel(), g["o"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1.ravel(), g["lse1"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l2.ravel(), g["lse2"], rtol=0, atol=1e-13)


# ---------------------------------------------------------------- I1 dense reductions

@pytest.mark.parametrize("grid", [(2, 4, 4), (3, 2, 5)])
def test_one_window_is_dense_attention(grid):
    inp = random_problem(11, 1, 2, 16, grid, grid, dtype=torch.float64)
    o, o1, _, l2, _ = oracle.squad_fwd(inp.q, inp.k, inp.v, grid, grid)
    ref = F.scaled_dot_product_attention(_f64(inp.q), _f64(inp.k), _f64(inp.v)).numpy()
    np.testing.assert_allclose(o1, ref, rtol=0, atol=1e-12)   # the local pass is dense attention
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)    # the global pass over m=1 is the identity
    own = (inp.q * inp.k).sum(-1).numpy() / math.sqrt(16)       # one key: lse2 is the own score
    np.testing.assert_allclose(l2, own, rtol=0, atol=1e-12)


@pytest.mark.parametrize("grid", [(2, 4, 4), (1, 3, 7)])
def test_one_token_windows_is_dense_attention(grid):
    inp = random_problem(12, 2, 1, 8, grid, (1, 1, 1), dtype=torch.float64)
    o, o1, _, _, _ = oracle.squad_fwd(inp.q, inp.k, inp.v, grid, (1, 1, 1))
    np.testing.assert_allclose(o1, inp.v.numpy(), rtol=0, atol=1e-13)  # w=1: local output is V
    ref = F.scaled_dot_product_attention(_f64(inp.q), _f64(inp.k), _f64(inp.v)).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_dense_reference_by_hand_2x2():
    # the library dense routine itself, against a 2-token case worked by hand
    q = torch.tensor([[[[1.0], [0.0]]]], dtype=torch.float64)
    k = torch.tensor([[[[0.0], [math.log(3.0)]]]], dtype=torch.float64)
    v = torch.tensor([[[[2.0], [6.0]]]], dtype=torch.float64)
    o = F.scaled_dot_product_attention(q, k, v, scale=1.0).ravel().tolist()
    assert abs(o[0] - (0.25 * 2 + 0.75 * 6)) < 1e-14   # query 1: weights 1/4, 3/4
    assert abs(o[1] - 4.0) < 1e-14                      # query 0 vector: equal weights


# ---------------------------------------------------------------- I2 masked brute force

@pytest.mark.parametrize("grid,tile,d", [
    ((4, 8, 8), (1, 4, 4), 64),     # the tiny workload's geometry
    ((4, 4, 6), (2, 2, 3), 16),     # tT > 1, non-square tiles
    ((3, 6, 4), (3, 1, 2), 8),
    ((2, 6, 10), (1, 3, 5), 12),
    ((5, 3, 3), (1, 3, 3), 5),
])
def test_two_pass_equals_block_masked_dense(grid, tile, d):
    inp = random_problem(21, 2, 2, d, grid, tile, dtype=torch.float64)
    o, o1, _, _, _ = oracle.squad_fwd(inp.q, inp.k, inp.v, grid, tile)
    ref_o, ref_o1 = _masked_sdpa_two_pass(_f64(inp.q), _f64(inp.k), _f64(inp.v), grid, tile)
    np.testing.assert_allclose(o1, ref_o1.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(o, ref_o.numpy(), rtol=0, atol=1e-12)


def test_explicit_scale_is_used():
    grid, tile = (2, 4, 4), (1, 2, 2)
    inp = random_problem(22, 1, 1, 8, grid, tile, dtype=torch.float64)
    o, _, _, _, _ = oracle.squad_fwd(inp.q, inp.k, inp.v, grid, tile, scale=0.7)
    ref, _ = _masked_sdpa_two_pass(inp.q, inp.k, inp.v, grid, tile, scale=0.7)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- I3 constant values

def test_constant_value_rows_pass_through():
    grid, tile = (4, 4, 4), (2, 2, 2)
    inp = random_problem(31, 1, 3, 8, grid, tile, dtype=torch.float64)
    c = np.linspace(-2.0, 3.0, 8)
    v = np.broadcast_to(c, inp.v.shape).copy()
    o, o1, _, _, _ = oracle.squad_fwd(inp.q, inp.k, v, grid, tile)
    np.testing.assert_allclose(o1, v, rtol=0, atol=1e-13)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- I4 permutation equivariance

def _token_perm(grid, tile, pos_perm=None, win_perm=None):
    """Token permutation that maps (window g, position r) to (win_perm[g], pos_perm[r])."""
    T, H, W = grid
    tT, tH, tW = tile
    nT, nH, nW = T // tT, H // tH, W // tW
    t, y, x = _coords(grid)
    g = np.ravel_multi_index((t // tT, y // tH, x // tW), (nT, nH, nW))
    r = np.ravel_multi_index((t % tT, y % tH, x % tW), (tT, tH, tW))
    if pos_perm is not None:
        r = pos_perm[r]
    if win_perm is not None:
        g = win_perm[g]
    gt, gy, gx = np.unravel_index(g, (nT, nH, nW))
    rt, ry, rx = np.unravel_index(r, (tT, tH, tW))
    return np.ravel_multi_index((gt * tT + rt, gy * tH + ry, gx * tW + rx), (T, H, W))


@pytest.mark.parametrize("which", ["positions", "windows"])
def test_permutation_equivariance(which):
    grid, tile = (4, 4, 6), (2, 2, 3)
    inp = random_problem(41, 1, 2, 8, grid, tile, dtype=torch.float64)
    rng = np.random.default_rng(0)
    w = 12
    m = 96 // w
    if which == "positions":
        pi = _token_perm(grid, tile, pos_perm=rng.permutation(w))
    else:
        pi = _token_perm(grid, tile, win_perm=rng.permutation(m))
    q, k, v = inp.q.numpy(), inp.k.numpy(), inp.v.numpy()
    qp, kp, vp = (np.empty_like(a) for a in (q, k, v))
    qp[:, :, pi], kp[:, :, pi], vp[:, :, pi] = q, k, v
    o, _, _, _, _ = oracle.squad_fwd(q, k, v, grid, tile)
    op, _, _, _, _ = oracle.squad_fwd(qp, kp, vp, grid, tile)
    np.testing.assert_allclose(op[:, :, pi], o, rtol=0, atol=1e-12)


def test_position_permutation_not_consistent_breaks_equivariance():
    # sanity of the previous test: permuting positions differently per window
    # changes the global groups, so the output must change
    grid, tile = (2, 4, 4), (1, 2, 2)
    inp = random_problem(42, 1, 1, 8, grid, tile, dtype=torch.float64)
    q, k, v = inp.q.numpy(), inp.k.numpy(), inp.v.numpy()
    pi = np.arange(32)
    pi[[0, 1]] = pi[[1, 0]]     # swap two tokens of the first window only
    qp, kp, vp = (np.empty_like(a) for a in (q, k, v))
    qp[:, :, pi], kp[:, :, pi], vp[:, :, pi] = q, k, v
    o, _, _, _, _ = oracle.squad_fwd(q, k, v, grid, tile)
    op, _, _, _, _ = oracle.squad_fwd(qp, kp, vp, grid, tile)
    assert np.abs(op[:, :, pi] - o).max() > 1e-3


# ---------------------------------------------------------------- I5 key-shift invariance

def test_key_shift_invariance_forward_and_backward():
    grid, tile = (2, 6, 4), (1, 3, 2)
    inp = random_problem(51, 1, 2, 8, grid, tile, dtype=torch.float64, with_do=True)
    b = 2.0 * np.random.default_rng(1).standard_normal(8)
    k2 = inp.k.numpy() + b
    o, _, _, _, _ = oracle.squad_fwd(inp.q, inp.k, inp.v, grid, tile)
    o2, _, _, _, _ = oracle.squad_fwd(inp.q, k2, inp.v, grid, tile)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    g1 = oracle.squad_bwd(inp.q, inp.k, inp.v, inp.do, grid, tile)
    g2 = oracle.squad_bwd(inp.q, k2, inp.v, inp.do, grid, tile)
    for a, b_ in zip(g1, g2):
        np.testing.assert_allclose(b_, a, rtol=0, atol=1e-11)


def test_large_logits_are_finite():
    # max-subtraction: logits of several hundred must not overflow exp
    grid, tile = (2, 4, 4), (1, 2, 2)
    inp = random_problem(52, 1, 1, 16, grid, tile, dtype=torch.float64)
    q = inp.q.numpy() * 40.0
    o, _, _, _, _ = oracle.squad_fwd(q, inp.k, inp.v, grid, tile)
    assert np.isfinite(o).all()
    ref, _ = _masked_sdpa_two_pass(torch.from_numpy(q), _f64(inp.k), _f64(inp.v), grid, tile)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-10)


# ---------------------------------------------------------------- I6 multiply-add count

@pytest.mark.parametrize("grid,tile", [((4, 8, 8), (1, 4, 4)), ((8, 16, 16), (2, 4, 8)), ((3, 4, 6), (3, 2, 1))])
def test_mac_count_closed_form(grid, tile):
    B, h, d = 1, 2, 8
    inp = random_problem(61, B, h, d, grid, tile, dtype=torch.float64)
    *_, macs = oracle.squad_fwd(inp.q, inp.k, inp.v, grid, tile)
    n = grid[0] * grid[1] * grid[2]
    w = tile[0] * tile[1] * tile[2]
    m = n // w
    assert macs == 2 * n * d * (w + m) * B * h
    assert 2 * macs < 4 * n * n * d * B * h or w == n or m == n   # sub-quadratic vs dense


# ---------------------------------------------------------------- I7 gradients

def _loss(q, k, v, do, grid, tile):
    o, *_ = oracle.squad_fwd(q, k, v, grid, tile, threads=1)
    return float((o * do).sum())


def test_backward_finite_differences():
    grid, tile = (2, 2, 4), (1, 2, 2)
    inp = random_problem(71, 1, 1, 3, grid, tile, dtype=torch.float64, with_do=True)
    q, k, v, do = (x.numpy().copy() for x in (inp.q, inp.k, inp.v, inp.do))
    dq, dk, dv = oracle.squad_bwd(q, k, v, do, grid, tile, threads=1)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            lp = _loss(q, k, v, do, grid, tile)
            x[idx] = old - h
            lm = _loss(q, k, v, do, grid, tile)
            x[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        err = np.abs(num - g).max() / max(1e-300, np.abs(num).max())
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("grid,tile", [((4, 8, 8), (1, 4, 4)), ((4, 4, 6), (2, 2, 3))])
def test_backward_matches_autograd_of_masked_dense(grid, tile):
    inp = random_problem(72, 2, 2, 8, grid, tile, dtype=torch.float64, with_do=True)
    q, k, v = (x.clone().requires_grad_(True) for x in (inp.q, inp.k, inp.v))
    o, _ = _masked_sdpa_two_pass(q, k, v, grid, tile)
    (o * inp.do).sum().backward()
    dq, dk, dv = oracle.squad_bwd(inp.q, inp.k, inp.v, inp.do, grid, tile)
    np.testing.assert_allclose(dq, q.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, k.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, v.grad.numpy(), rtol=0, atol=1e-11)


def _random_geometries(count, seed):
    """Seeded grids (each side 1..9) with a random divisor of each side as the window tile."""
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < count:
        grid = tuple(int(x) for x in rng.integers(1, 10, size=3))
        if math.prod(grid) > 360:
            continue
        tile = tuple(int(rng.choice([t for t in range(1, g + 1) if g % t == 0])) for g in grid)
        out.append((grid, tile, int(rng.integers(1, 9))))
    return out


@pytest.mark.parametrize("grid,tile,d", _random_geometries(24, 20261203))
def test_forward_and_backward_equal_masked_dense_on_random_geometries(grid, tile, d):
    # a sweep over seeded random grids and tiles (windows of one token, whole-grid windows,
    # tT > 1, odd sides): forward against the masked library SDPA, backward against autograd
    inp = random_problem(73, 1, 2, d, grid, tile, dtype=torch.float64, with_do=True)
    q, k, v = (x.clone().requires_grad_(True) for x in (inp.q, inp.k, inp.v))
    ref_o, ref_o1 = _masked_sdpa_two_pass(q, k, v, grid, tile)
    (ref_o * inp.do).sum().backward()
    o, o1, _, _, _ = oracle.squad_fwd(inp.q, inp.k, inp.v, grid, tile)
    np.testing.assert_allclose(o1, ref_o1.detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(o, ref_o.detach().numpy(), rtol=0, atol=1e-12)
    dq, dk, dv = oracle.squad_bwd(inp.q, inp.k, inp.v, inp.do, grid, tile)
    for name, got, t in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        np.testing.assert_allclose(got, t.grad.numpy(), rtol=0, atol=1e-11, err_msg=name)


def test_bad_shapes_rejected():
    inp = random_problem(81, 1, 1, 4, (2, 4, 4), (1, 2, 2), dtype=torch.float64)
    with pytest.raises(ValueError):
        oracle.squad_fwd(inp.q, inp.k, inp.v, (2, 4, 4), (1, 3, 2))   # 3 does not divide 4
    with pytest.raises(ValueError):
        oracle.squad_fwd(inp.q, inp.k, inp.v, (2, 4, 5), (1, 2, 1))   # n != T*H*W
