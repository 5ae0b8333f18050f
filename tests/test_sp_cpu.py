"""Sequence-parallel forward on the CPU: the library's plan (index maps) and the exchange.

The plan functions of libsquad (squad_sp_plan_info / squad_sp_plan_maps) are host
code and run here without a GPU. Two checks:
  - routing: every rank's maps, applied to token ids and exchanged as the all-to-all
    would, put each token's row where the plan says (position-major: row
    pos * m + g holds the token of window g at position pos) and bring every row
    back to its owner in token order, for uneven splits of frames and positions;
  - the forward over gloo (world sizes 2 and 3): each rank holds its frames, runs
    the local pass and the global pass with the fp64 oracle, exchanges rows with
    torch.distributed.all_to_all_single in the library's layout, and the gathered
    output equals the oracle on the whole problem.
The pack/unpack layout emulated here is the one include/squad.h documents for
squad_sp_pack / squad_sp_unpack; the GPU tests check the kernels against it.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _plan(grid, tile, G, rank, B=1, heads=1, d=32):
    from sub_quadratic_two_b200.sp import SpPlan
    return SpPlan(B, heads, d, grid, tile, G, rank, dtype=torch.float32)


def np_pack(srcs, idx, counts):
    """[peer][tensor][slice][counts[peer]] rows (srcs: [slices, rows_in, d] arrays)."""
    pref = np.concatenate([[0], np.cumsum(counts)])
    parts = []
    for q in range(len(counts)):
        for t in srcs:
            parts.append(t[:, idx[pref[q]:pref[q + 1]], :].reshape(-1, t.shape[-1]))
    return np.concatenate(parts)


def np_unpack(buf, ntensors, slices, rows_out, src_rank, src_row, counts):
    pref = np.concatenate([[0], np.cumsum(counts)])
    cnt = np.asarray(counts)[src_rank]
    outs = []
    for t in range(ntensors):
        s = np.arange(slices)[:, None]
        rows = ntensors * slices * pref[src_rank][None, :] + (t * slices + s) * cnt[None, :] + src_row[None, :]
        outs.append(buf[rows])
    return outs


def _token(grid, tile, g, pos):
    T, H, W = grid
    tT, tH, tW = tile
    nH, nW = H // tH, W // tW
    fw, wh, ww = g // (nH * nW), (g // nW) % nH, g % nW
    pt, ph, pw = pos // (tH * tW), (pos // tW) % tH, pos % tW
    return ((fw * tT + pt) * H + wh * tH + ph) * W + ww * tW + pw


@pytest.mark.parametrize("grid,tile,G", [
    ((31, 22, 40), (1, 11, 20), 8),   # the 27,280-token grid: 31 frames and 220 positions over 8 ranks
    ((31, 22, 40), (1, 11, 20), 3),
    ((6, 4, 6), (2, 2, 3), 1),
    ((6, 4, 6), (2, 2, 3), 2),
    ((10, 4, 4), (2, 2, 2), 5),       # 5 frame windows, 8 positions over 5 ranks
    ((9, 6, 4), (3, 3, 2), 3),        # tT > 1, one frame window per rank
])
def test_plan_routes_every_row(grid, tile, G):
    T, H, W = grid
    plans = [_plan(grid, tile, G, r) for r in range(G)]
    n = T * H * W
    assert sum(p.n_local for p in plans) == n
    assert [p.t0 for p in plans] == list(np.cumsum([0] + [p.T for p in plans])[:-1])
    # each rank's shard: the token ids of its frames, as one slice of one-element rows
    shard = [np.arange(p.t0 * H * W, (p.t0 + p.T) * H * W, dtype=np.float64)[None, :, None] for p in plans]
    sends = [np_pack([shard[r]], plans[r].send1, plans[r].send1_count) for r in range(G)]
    for r, p in enumerate(plans):
        assert sorted(p.send1.tolist()) == list(range(p.n_local))      # every local row sent once
        # what rank r receives: source after source, the chunk each source built for r
        offs = [np.concatenate([[0], np.cumsum(plans[s].send1_count)]) for s in range(G)]
        recv = np.concatenate([sends[s][offs[s][r]:offs[s][r + 1]] for s in range(G)])
        assert [len(sends[s][offs[s][r]:offs[s][r + 1]]) for s in range(G)] == list(p.recv1_count)
        (pm,) = np_unpack(recv, 1, 1, p.n_pos, p.recv1_src, p.recv1_row, p.recv1_count)
        want = [_token(grid, tile, g, p.p0 + pi) for pi in range(p.np_) for g in range(p.m)]
        assert pm[0, :, 0].astype(np.int64).tolist() == want
        p.pm = pm
    sends2 = [np_pack([plans[r].pm], plans[r].send2, plans[r].send2_count) for r in range(G)]
    for r, p in enumerate(plans):
        offs = [np.concatenate([[0], np.cumsum(plans[s].send2_count)]) for s in range(G)]
        recv = np.concatenate([sends2[s][offs[s][r]:offs[s][r + 1]] for s in range(G)])
        (back,) = np_unpack(recv, 1, 1, p.n_local, p.recv2_src, p.recv2_row, p.recv2_count)
        assert np.array_equal(back, shard[r])


def test_plan_rejects_more_ranks_than_frame_windows():
    from sub_quadratic_two_b200 import SquadError
    with pytest.raises(SquadError):
        _plan((4, 4, 4), (2, 2, 2), 3, 0)   # 2 frame windows cannot feed 3 ranks


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _sp_worker(rank, G, port, grid, tile, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import oracle
    from workloads import random_problem
    dist.init_process_group("gloo", rank=rank, world_size=G)
    try:
        B, heads, d = 2, 2, 32
        full = random_problem(81, B, heads, d, grid, tile, dtype=torch.float64)
        p = _plan(grid, tile, G, rank, B, heads, d)
        T, H, W = grid
        lo, hi = p.t0 * H * W, (p.t0 + p.T) * H * W
        q, k, v = (x[:, :, lo:hi].numpy() for x in (full.q, full.k, full.v))
        S = B * heads
        _, o1, _, _, _ = oracle.squad_fwd(q, k, v, p.local_grid, p.tile)          # local pass of the shard
        flat = [x.reshape(S, p.n_local, d) for x in (q, k, o1)]
        send = torch.from_numpy(np_pack(flat, p.send1, p.send1_count))
        recv = torch.empty((int(p.recv1_count.sum()) * 3 * S, d), dtype=torch.float64)
        dist.all_to_all_single(recv, send, [int(c) * 3 * S for c in p.recv1_count],
                               [int(c) * 3 * S for c in p.send1_count])
        qg, kg, o1g = (x.reshape(B, heads, p.n_pos, d)
                       for x in np_unpack(recv.numpy(), 3, S, p.n_pos, p.recv1_src, p.recv1_row, p.recv1_count))
        _, og, _, _, _ = oracle.squad_fwd(qg, kg, o1g, p.global_grid, p.global_tile)   # global pass of its positions
        send2 = torch.from_numpy(np_pack([og.reshape(S, p.n_pos, d)], p.send2, p.send2_count))
        recv2 = torch.empty((int(p.recv2_count.sum()) * S, d), dtype=torch.float64)
        dist.all_to_all_single(recv2, send2, [int(c) * S for c in p.recv2_count], [int(c) * S for c in p.send2_count])
        (o,) = np_unpack(recv2.numpy(), 1, S, p.n_local, p.recv2_src, p.recv2_row, p.recv2_count)
        ref, _, _, _, _ = oracle.squad_fwd(full.q, full.k, full.v, grid, tile)
        err = float(np.abs(o.reshape(B, heads, p.n_local, d) - ref[:, :, lo:hi]).max())
        out.put((rank, err))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("G,grid,tile", [(2, (5, 4, 6), (1, 2, 3)), (3, (7, 4, 4), (1, 2, 2))])
def test_sp_forward_over_gloo_matches_the_oracle(G, grid, tile):
    port = _free_port()
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    procs = [ctx.Process(target=_sp_worker, args=(r, G, port, grid, tile, qu)) for r in range(G)]
    for p in procs:
        p.start()
    res = sorted(qu.get(timeout=240) for _ in range(G))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _ in res] == list(range(G))
    for rank, err in res:
        assert err <= 1e-12, (rank, err)
