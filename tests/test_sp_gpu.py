"""Sequence-parallel forward on one GPU: the shuffle kernels and an emulated exchange.

squad_sp_pack / squad_sp_unpack must produce exactly the layout include/squad.h
documents (checked against the numpy emulation of tests/test_sp_cpu.py), and an
out-of-range index must be skipped and reported (SQUAD_ERR_INDEX), not followed.
Then G ranks are emulated one after another on this GPU: each runs its local pass,
packs, the all-to-all is emulated by handing each rank the chunks the others built
for it, and so on through the global pass and the way back; the gathered output
must equal squad_attn_fwd on the whole problem (the same kernels compute every row)
and the fp64 oracle within the bf16 bounds. Multi-GPU runs need NCCL and more than
one GPU and are not part of these tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sub_quadratic_two_b200 as sq
from sub_quadratic_two_b200.sp import SpPlan, sp_pack, sp_unpack
from test_sp_cpu import np_pack, np_unpack
from workloads import random_problem

pytestmark = pytest.mark.gpu


def test_pack_and_unpack_kernels_give_the_documented_layout(cuda_ok):
    g = torch.Generator().manual_seed(3)
    B, h, rows_in, d = 2, 3, 37, 64
    srcs = [torch.randn(B, h, rows_in, d, generator=g).to(torch.bfloat16) for _ in range(3)]
    counts = np.array([5, 0, 11, 7], dtype=np.int32)
    idx = torch.randint(0, rows_in, (int(counts.sum()),), generator=g, dtype=torch.int32)
    got = sp_pack([s.cuda() for s in srcs], idx.cuda(), counts)
    want = np_pack([s.reshape(B * h, rows_in, d).float().numpy() for s in srcs], idx.numpy(), counts)
    assert np.array_equal(got.float().cpu().numpy(), want)
    rows_out = 29
    src_rank = torch.randint(0, 4, (rows_out,), generator=g, dtype=torch.int32)
    src_rank[src_rank == 1] = 2                      # peer 1 sent nothing
    src_row = torch.tensor([int(torch.randint(0, int(counts[q]), (1,), generator=g)) for q in src_rank.tolist()],
                           dtype=torch.int32)
    outs = sp_unpack(got, 3, B, h, rows_out, src_rank.cuda(), src_row.cuda(), counts)
    sq.poll_device_error()
    want_u = np_unpack(want, 3, B * h, rows_out, src_rank.numpy(), src_row.numpy(), counts)
    for o, w in zip(outs, want_u):
        assert np.array_equal(o.float().cpu().numpy().reshape(B * h, rows_out, d), w)


def test_out_of_range_indices_are_reported_not_followed(cuda_ok):
    src = torch.randn(1, 1, 8, 32, device="cuda")
    counts = np.array([4], dtype=np.int32)
    idx = torch.tensor([0, 1, 8, 3], dtype=torch.int32, device="cuda")    # 8 is past the 8 rows
    out = sp_pack([src], idx, counts)
    with pytest.raises(sq.SquadError) as e:
        sq.poll_device_error()
    assert e.value.status == 8                                           # SQUAD_ERR_INDEX
    assert torch.equal(out[[0, 1, 3]], src[0, 0, [0, 1, 3]])
    rank = torch.tensor([0, 0, 1], dtype=torch.int32, device="cuda")    # peer 1 does not exist
    row = torch.tensor([0, 3, 0], dtype=torch.int32, device="cuda")
    (back,) = sp_unpack(out, 1, 1, 1, 3, rank, row, counts)
    with pytest.raises(sq.SquadError) as e:
        sq.poll_device_error()
    assert e.value.status == 8
    sq.poll_device_error()                                               # the word was cleared


def _emulated_sp_forward(q, k, v, grid, tile, G):
    """Every rank's steps on this GPU; the all-to-alls are emulated by slicing chunks."""
    B, h, n, d = q.shape
    T, H, W = grid
    plans = [SpPlan(B, h, d, grid, tile, G, r) for r in range(G)]
    S = B * h

    def exchange(sends, send_counts, ntensors):
        out = []
        for r in range(G):
            chunks = []
            for s in range(G):
                off = np.concatenate([[0], np.cumsum(send_counts[s])]) * ntensors * S
                chunks.append(sends[s][int(off[r]):int(off[r + 1])])
            out.append(torch.cat(chunks))
        return out

    shards, sends = [], []
    for r, p in enumerate(plans):
        lo, hi = p.t0 * H * W, (p.t0 + p.T) * H * W
        qs, ks, vs = (x[:, :, lo:hi].contiguous() for x in (q, k, v))
        o1 = torch.empty_like(qs)
        sq.squad_attn_fwd_pass(1, qs, ks, vs, o1, p.local_grid, p.tile)
        shards.append((lo, hi))
        sends.append(sp_pack([qs, ks, o1], p.device_maps(q.device)["send1"], p.send1_count))
    recvs = exchange(sends, [p.send1_count for p in plans], 3)
    sends2 = []
    for r, p in enumerate(plans):
        m = p.device_maps(q.device)
        qg, kg, o1g = sp_unpack(recvs[r], 3, B, h, p.n_pos, m["recv1_src"], m["recv1_row"], p.recv1_count)
        og = torch.empty_like(qg)
        sq.squad_attn_fwd_pass(1, qg, kg, o1g, og, p.global_grid, p.global_tile)
        sends2.append(sp_pack([og], m["send2"], p.send2_count))
    recvs2 = exchange(sends2, [p.send2_count for p in plans], 1)
    o = torch.empty_like(q)
    for r, p in enumerate(plans):
        m = p.device_maps(q.device)
        (orow,) = sp_unpack(recvs2[r], 1, B, h, p.n_local, m["recv2_src"], m["recv2_row"], p.recv2_count)
        lo, hi = shards[r]
        o[:, :, lo:hi] = orow
    sq.poll_device_error()
    return o


@pytest.mark.parametrize("grid,tile,heads,G", [
    ((31, 22, 40), (1, 11, 20), 2, 3),    # 27,280 tokens: 31 frames over 3 ranks (11, 10, 10)
    ((9, 12, 16), (3, 4, 8), 2, 2),       # tT > 1: three frame windows over 2 ranks
    ((8, 16, 16), (2, 4, 8), 1, 4),       # 64 positions over 4 ranks
])
def test_emulated_ranks_equal_the_single_gpu_forward(cuda_ok, grid, tile, heads, G):
    inp = random_problem(91, 1, heads, 128, grid, tile, dtype=torch.bfloat16)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    o = _emulated_sp_forward(q, k, v, grid, tile, G)
    ref, *_ = sq.squad_attn_fwd(q, k, v, grid, tile, save=False)
    sq.poll_device_error()
    assert torch.equal(o, ref)
    ro, *_ = oracle.squad_fwd(inp.q[:, :1], inp.k[:, :1], inp.v[:, :1], grid, tile)
    e = (o[:, :1].double().cpu() - torch.from_numpy(ro)).abs()
    assert e.max().item() <= 1.5e-2 and e.mean().item() <= 2e-3
