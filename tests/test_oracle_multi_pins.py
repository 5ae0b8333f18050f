"""Pins for the oracle's k-pass functions (passes over nested tiles).

The pages name composing more than two passes as an outlook ("SQuad: Sub-Quadratic
Attention Distillation for Efficient Video Generation", gist.science technical
summary, Significance and Claims). Reading: nested tiles t_1 | ... | t_{k-1} | grid;
pass j attends among tokens in the same t_j-window at the same position inside
their t_{j-1}-window (t_0 = one token, t_k = the grid), values = previous output.
Each check below comes from outside the k-pass code: the two-pass oracle (pinned on
its own), dense attention from torch's SDPA, dense attention with boolean masks
built from coordinates in numpy, a closed-form multiply-add count, and finite
differences.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from workloads import random_problem


def _coords(grid):
    T, H, W = grid
    return np.unravel_index(np.arange(T * H * W), (T, H, W))  # x fastest


def _pass_masks(grid, tiles):
    """Boolean [n, n] masks of every pass, from token coordinates."""
    c = np.stack(_coords(grid), 1)
    chain = [(1, 1, 1)] + [tuple(t) for t in tiles] + [tuple(grid)]
    masks = []
    for inner, outer in zip(chain[:-1], chain[1:]):
        win = c // np.array(outer)
        pos = c % np.array(inner)
        same = (win[:, None, :] == win[None, :, :]).all(-1) & (pos[:, None, :] == pos[None, :, :]).all(-1)
        masks.append(torch.from_numpy(same))
    return masks


def _masked_dense_passes(q, k, v, grid, tiles):
    val = v
    for m in _pass_masks(grid, tiles):
        val = F.scaled_dot_product_attention(q, k, val, attn_mask=m)
    return val


def _problem(seed, grid, d=16, heads=2, B=1):
    inp = random_problem(seed, B, heads, d, grid, (1, 1, 1), dtype=torch.float64, with_do=True)
    return inp.q, inp.k, inp.v, inp.do


def test_one_tile_is_the_two_pass_operator():
    grid, tile = (2, 4, 6), (1, 2, 3)
    q, k, v, do = _problem(1, grid)
    o, inter, lse, _ = oracle.squad_fwd_multi(q, k, v, grid, [tile])
    ro, ro1, rl1, rl2, _ = oracle.squad_fwd(q, k, v, grid, tile)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-13)
    np.testing.assert_allclose(inter[0], ro1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[0], rl1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[1], rl2, rtol=0, atol=1e-13)
    g = oracle.squad_bwd_multi(q, k, v, do, grid, [tile])
    r = oracle.squad_bwd(q, k, v, do, grid, tile)
    for a, b in zip(g, r):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_trivial_inner_tile_reduces_to_two_passes():
    # t_1 = one token: pass 1 is the identity (O1 = V), passes 2 and 3 are SQuad with t_2
    grid, tile = (2, 4, 8), (2, 2, 4)
    q, k, v, _ = _problem(2, grid)
    o, inter, _, _ = oracle.squad_fwd_multi(q, k, v, grid, [(1, 1, 1), tile])
    ro, _, _, _, _ = oracle.squad_fwd(q, k, v, grid, tile)
    np.testing.assert_allclose(inter[0], v.numpy(), rtol=0, atol=1e-15)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)


def test_outer_tile_equal_to_grid_reduces_to_two_passes():
    # t_2 = grid: the last pass groups single tokens (identity)
    grid, tile = (2, 4, 8), (1, 2, 4)
    q, k, v, _ = _problem(3, grid)
    o, inter, _, _ = oracle.squad_fwd_multi(q, k, v, grid, [tile, grid])
    ro, _, _, _, _ = oracle.squad_fwd(q, k, v, grid, tile)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(o, inter[1], rtol=0, atol=1e-15)


def test_trivial_tiles_give_dense_attention():
    grid = (2, 3, 4)
    q, k, v, _ = _problem(4, grid)
    o, _, _, _ = oracle.squad_fwd_multi(q, k, v, grid, [(1, 1, 1), (1, 1, 1)])
    ref = F.scaled_dot_product_attention(q, k, v)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("grid,tiles", [
    ((2, 4, 8), [(1, 2, 2), (2, 2, 4)]),
    ((4, 4, 4), [(1, 1, 2), (2, 2, 2)]),
    ((3, 6, 4), [(1, 3, 1), (3, 3, 2)]),
    ((2, 4, 8), [(1, 1, 2), (1, 2, 2), (2, 2, 4)]),  # four passes
])
def test_passes_equal_masked_dense_attention(grid, tiles):
    q, k, v, _ = _problem(5, grid)
    o, _, _, _ = oracle.squad_fwd_multi(q, k, v, grid, tiles)
    ref = _masked_dense_passes(q, k, v, grid, tiles)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)


def _random_chains(count, seed):
    """Seeded grids (sides 1..8) with chains of 1-3 nested tiles (each a divisor chain)."""
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < count:
        grid = tuple(int(x) for x in rng.integers(1, 9, size=3))
        if int(np.prod(grid)) > 256:
            continue
        ntiles = int(rng.integers(1, 4))
        tiles, cur = [], (1, 1, 1)
        for _ in range(ntiles):
            # the next tile: a multiple of the current one that divides the grid
            nxt = tuple(int(rng.choice([t for t in range(c, g + 1) if t % c == 0 and g % t == 0]))
                        for c, g in zip(cur, grid))
            tiles.append(nxt)
            cur = nxt
        out.append((grid, tiles, int(rng.integers(1, 7))))
    return out


@pytest.mark.parametrize("grid,tiles,d", _random_chains(16, 1203))
def test_random_chains_equal_masked_dense_forward_and_backward(grid, tiles, d):
    # seeded random grids and tile chains (repeated tiles, one-token tiles, whole-grid
    # tiles): forward against masked SDPA composed pass by pass, backward against autograd
    q, k, v, do = _problem(8, grid, d=d)
    qq, kk, vv = (t.clone().requires_grad_(True) for t in (q, k, v))
    ref = _masked_dense_passes(qq, kk, vv, grid, tiles)
    (ref * do).sum().backward()
    o, _, _, _ = oracle.squad_fwd_multi(q, k, v, grid, tiles)
    np.testing.assert_allclose(o, ref.detach().numpy(), rtol=0, atol=1e-12)
    g = oracle.squad_bwd_multi(q, k, v, do, grid, tiles)
    for name, a, b in zip(("dq", "dk", "dv"), g, (qq.grad, kk.grad, vv.grad)):
        np.testing.assert_allclose(a, b.numpy(), rtol=0, atol=1e-11, err_msg=name)


def test_mac_count_closed_form():
    # 2 n d sum_j |t_j| / |t_{j-1}| per (batch, head): scores plus value sums
    grid, tiles = (2, 4, 8), [(1, 2, 2), (2, 2, 4)]
    q, k, v, _ = _problem(6, grid, d=8, heads=3, B=2)
    _, _, _, macs = oracle.squad_fwd_multi(q, k, v, grid, tiles)
    n = 64
    sizes = [1, 4, 16, n]
    expect = 2 * 3 * 2 * n * 8 * sum(b // a for a, b in zip(sizes[:-1], sizes[1:]))
    assert macs == expect


def test_backward_matches_autograd_of_masked_dense():
    grid, tiles = (2, 4, 4), [(1, 2, 1), (2, 2, 2)]
    q, k, v, do = _problem(7, grid, d=8)
    qq, kk, vv = (t.clone().requires_grad_(True) for t in (q, k, v))
    (_masked_dense_passes(qq, kk, vv, grid, tiles) * do).sum().backward()
    g = oracle.squad_bwd_multi(q, k, v, do, grid, tiles)
    for a, b in zip(g, (qq.grad, kk.grad, vv.grad)):
        np.testing.assert_allclose(a, b.numpy(), rtol=0, atol=1e-11)


def test_backward_finite_differences():
    grid, tiles = (2, 2, 4), [(1, 1, 2), (2, 1, 2)]
    q, k, v, do = _problem(8, grid, d=4, heads=1)
    dq, dk, dv = oracle.squad_bwd_multi(q, k, v, do, grid, tiles)
    loss = lambda q_, k_, v_: float((oracle.squad_fwd_multi(q_, k_, v_, grid, tiles)[0] * do.numpy()).sum())
    eps = 1e-6
    rng = np.random.default_rng(0)
    for grad, which in ((dq, 0), (dk, 1), (dv, 2)):
        for _ in range(4):
            idx = tuple(int(rng.integers(0, s)) for s in q.shape)
            args = [q.clone(), k.clone(), v.clone()]
            args[which][idx] += eps
            up = loss(*args)
            args[which][idx] -= 2 * eps
            dn = loss(*args)
            assert abs((up - dn) / (2 * eps) - grad[idx]) < 1e-6


def test_tiles_that_do_not_nest_are_rejected():
    q, k, v, _ = _problem(9, (2, 4, 8))
    for tiles in ([(1, 3, 1)], [(1, 2, 4), (1, 4, 2)], [(2, 2, 2), (1, 1, 1)]):
        with pytest.raises(ValueError):
            oracle.squad_fwd_multi(q, k, v, (2, 4, 8), tiles)


@pytest.mark.parametrize("grid,tiles", [
    ((2, 4, 6), [(1, 2, 3)]),
    ((2, 4, 8), [(1, 1, 2), (1, 2, 4)]),
    ((4, 4, 4), [(1, 1, 2), (2, 2, 2), (2, 4, 4)]),
])
def test_uniform_scores_give_the_mean_of_v(grid, tiles):
    # With Q = 0 every score is 0 and every softmax is uniform over its group. Pass 1
    # then gives each token the mean of V over its t_1-window; pass j averages those
    # window means over the t_{j-1}-windows inside a t_j-window, i.e. the mean of V over
    # the t_j-window; the last pass gives the mean of V over the whole grid, for every
    # token. Each LSE is log of the pass's group size.
    q, k, v, _ = _problem(11, grid, d=8)
    q = torch.zeros_like(q)
    o, inter, lse, _ = oracle.squad_fwd_multi(q, k, v, grid, tiles)
    vn = v.numpy()
    want = np.broadcast_to(vn.mean(axis=2, keepdims=True), vn.shape)
    np.testing.assert_allclose(o, want, rtol=0, atol=1e-12)
    # intermediate j: mean of V over the token's t_j-window
    T, H, W = grid
    t, y, x = _coords(grid)
    for j, tile in enumerate(tiles):
        win = ((t // tile[0]) * (H // tile[1]) + y // tile[1]) * (W // tile[2]) + x // tile[2]
        exp = np.zeros_like(vn)
        for wdx in np.unique(win):
            sel = win == wdx
            exp[:, :, sel, :] = vn[:, :, sel, :].mean(axis=2, keepdims=True)
        np.testing.assert_allclose(inter[j], exp, rtol=0, atol=1e-12)
    chain = [(1, 1, 1)] + [tuple(tl) for tl in tiles] + [tuple(grid)]
    for j, (inner, outer) in enumerate(zip(chain[:-1], chain[1:])):
        size = np.prod(outer) // np.prod(inner)
        np.testing.assert_allclose(lse[j], np.log(size), rtol=0, atol=1e-12)
