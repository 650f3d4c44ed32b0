"""Host logic of the multi-GPU Star path (block_sparse_long_rope_b200.sharded)
on CPU with gloo ranks: the shard plan, the query broadcast and the
all-gather of partial slots, checked end to end against the oracle. Each
rank packs the oracle's partials of its own splits exactly as the kernels
write them; the gathered slots, read by the layout star_lse_merge_ranks
documents and merged by the oracle, must give global attention [pith
2WVXFXZ2, Referee summary: local outputs and softmax statistics re-weighted
at the query host]."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_long_rope_b200 import sharded


@pytest.mark.parametrize("L,b,world", [(96, 16, 2), (96, 16, 3), (100, 16, 4), (64, 64, 1),
                                       (16384, 4096, 4), (131072, 32768, 3)])
def test_shard_plan_covers_every_block_once(L, b, world):
    plan = sharded.shard_plan(L, b, world)
    n = -(-L // b)
    assert [s.rank for s in plan] == list(range(world))
    assert plan[0].first_block == 0 and plan[-1].last_block == n
    for s, t in zip(plan, plan[1:]):
        assert s.last_block == t.first_block
    assert all(s.n_local >= 1 for s in plan)
    assert max(s.n_local for s in plan) - min(s.n_local for s in plan) <= 1
    assert sum(s.rows for s in plan) == L
    assert all(s.row0 == s.first_block * b for s in plan)
    assert [s.query_host for s in plan] == [False] * (world - 1) + [True]
    assert sum(s.nsplit for s in plan) == n + 1
    order = sharded.global_split_order(plan)
    assert len(order) == n + 1 and order[-1] == (world - 1, plan[-1].n_local)


def test_shard_plan_rejects_more_ranks_than_blocks():
    with pytest.raises(ValueError):
        sharded.shard_plan(100, 50, 3)


def test_anchor_table_gives_every_local_block_the_anchor():
    s = sharded.shard_plan(16384, 4096, 2)[1]
    src, pos, bounds = sharded.anchor_table(s, 4096)
    assert (src == -1 - np.arange(4096)).all() and (pos == np.arange(4096)).all()
    assert bounds.shape == (2, 2) and (bounds == (0, 4096)).all()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASE = dict(B=1, L=96, b=16, Hq=4, Hkv=2, D=8, T=2, tail=3, theta=1e4)


def _inputs():
    c = CASE
    g = torch.Generator().manual_seed(7)
    q = torch.randn(c["B"], c["T"], c["Hq"], c["D"], generator=g).to(torch.bfloat16)
    kc = torch.randn(c["B"], c["L"], c["Hkv"], c["D"], generator=g).to(torch.bfloat16)
    vc = torch.randn(c["B"], c["L"], c["Hkv"], c["D"], generator=g).to(torch.bfloat16)
    kt = torch.randn(c["B"], c["tail"] + c["T"], c["Hkv"], c["D"], generator=g).to(torch.bfloat16)
    vt = torch.randn(c["B"], c["tail"] + c["T"], c["Hkv"], c["D"], generator=g).to(torch.bfloat16)
    return q, kc, vc, kt, vt


def _rows():
    c = CASE
    bb, hh, tt = np.meshgrid(np.arange(c["B"]), np.arange(c["Hq"]), np.arange(c["T"]), indexing="ij")
    return bb.ravel(), hh.ravel(), tt.ravel()


def _rank(rank, world, port, out):
    from oracle import oracle as orc

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c = CASE
        B, Hq, D, T = c["B"], c["Hq"], c["D"], c["T"]
        q, kc, vc, kt, vt = _inputs()
        plan = sharded.shard_plan(c["L"], c["b"], world)
        s = plan[rank]
        n = -(-c["L"] // c["b"])
        # the query host holds the new tokens; the broadcast hands them out
        qbuf = q.clone() if s.query_host else torch.zeros_like(q)
        sharded.broadcast_query(qbuf, plan)
        assert torch.equal(qbuf, q)
        # this rank's partials (its blocks; the tail on the query host), packed
        # densely [B, Hq, nsplit, T, D] at the start of an S-slot send buffer
        qb, qh, qt = _rows()
        po, pl = orc.phase2_rows(qbuf, kc, vc, kt, vt, c["b"], c["tail"], c["theta"], qb, qh, qt)
        mine = list(range(s.first_block, s.last_block)) + ([n] if s.query_host else [])
        S = max(p.nsplit for p in plan)
        dense_o = po[:, mine, :].reshape(B, Hq, T, len(mine), D).transpose(0, 1, 3, 2, 4)
        dense_l = pl[:, mine].reshape(B, Hq, T, len(mine)).transpose(0, 1, 3, 2)
        slot_o, slot_l = B * Hq * S * T * D, B * Hq * S * T
        send_o = torch.full((slot_o,), float("nan"))
        send_l = torch.full((slot_l,), float("nan"))   # unused slots must be ignored
        send_o[:dense_o.size] = torch.from_numpy(np.ascontiguousarray(dense_o).ravel()).float()
        send_l[:dense_l.size] = torch.from_numpy(np.ascontiguousarray(dense_l).ravel()).float()
        recv_o = torch.empty(world * slot_o)
        recv_l = torch.empty(world * slot_l)
        sharded.exchange_partials(send_o, send_l, recv_o, recv_l, slot_o, slot_l, world)
        # read the slots by the documented layout, merge in rank order
        segs_o, segs_l = [], []
        for r, p in enumerate(plan):
            m = p.nsplit
            segs_o.append(recv_o[r * slot_o:r * slot_o + B * Hq * m * T * D].view(B, Hq, m, T, D))
            segs_l.append(recv_l[r * slot_l:r * slot_l + B * Hq * m * T].view(B, Hq, m, T))
        allo = torch.cat(segs_o, dim=2).permute(0, 1, 3, 2, 4).reshape(B * Hq * T, n + 1, D)
        alll = torch.cat(segs_l, dim=2).permute(0, 1, 3, 2).reshape(B * Hq * T, n + 1)
        mo, ml = orc.lse_merge(allo.double().numpy(), alll.double().numpy())
        go, gl = orc.global_rows(q, kc, vc, kt, vt, c["tail"], c["theta"], qb, qh, qt)
        out.put((rank, float(np.abs(mo - go).max()), float(np.abs(ml - gl).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_exchange_and_merge_equal_global_attention(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = [out.get(timeout=10) for _ in range(world)]
    assert sorted(r for r, _, _ in res) == list(range(world))
    for _, eo, el in res:
        assert eo < 1e-6 and el < 1e-6  # fp32 partials, exact merge
