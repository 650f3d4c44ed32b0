"""Star Attention with one sequence's context blocks spread over several
GPUs, one process per GPU (torch.distributed, NCCL over NVLink).

This is the pages' own deployment [pith 2WVXFXZ2, "What carries the
argument" and Referee summary]:
- Phase 1 needs no communication. Every host encodes its blocks, each
  prefixed with the anchor block c_1 at its original positions 0..a-1. A
  rank without block 0 receives the anchor's K/V input rows with its own
  rows, as every host receives c_1 with its block.
- Phase 2 broadcasts the query from the query host. Every rank computes one
  partial (output, LSE) per local block over its own KV cache, and the query
  host also computes the causal tail split, which holds the query and
  response tokens' KV. An all-gather of the partials gives every rank the
  exact merge. KV caches never move.

Ranks own contiguous runs of blocks; the last rank is the query host, so the
tail follows its context rows in its cache. All compute runs in the C-ABI
kernels (star_phase1_encode[_ext], star_phase2_partial_ext,
star_lse_merge_ranks); this module holds the plan and the collectives.
"""
from dataclasses import dataclass

import numpy as np
import torch

from . import star
from .configs import Workload


@dataclass(frozen=True)
class Shard:
    rank: int
    world: int
    first_block: int   # global index of the shard's first context block
    last_block: int    # one past its last block
    row0: int          # global row (= position) of its first context row
    rows: int          # context rows it holds
    query_host: bool   # holds the tail (query and response tokens)

    @property
    def n_local(self):
        return self.last_block - self.first_block

    @property
    def nsplit(self):
        return self.n_local + (1 if self.query_host else 0)


def shard_plan(L, block_len, world):
    """Contiguous runs of blocks per rank, as even as possible (earlier ranks
    take the extra block); the last rank is the query host."""
    n = -(-L // block_len)
    if world < 1 or world > n:
        raise ValueError(f"{world} ranks for {n} blocks: every rank needs a block")
    base, extra = divmod(n, world)
    plan, first = [], 0
    for r in range(world):
        cnt = base + (1 if r < extra else 0)
        last = first + cnt
        row0 = first * block_len
        plan.append(Shard(r, world, first, last, row0, min(last * block_len, L) - row0,
                          r == world - 1))
        first = last
    return plan


def anchor_table(shard, anchor_len):
    """Prefix table of a shard without block 0: the anchor as given rows
    (extra_k/v rows 0..a-1) at positions 0..a-1, seen by every local block."""
    src = -1 - np.arange(anchor_len, dtype=np.int32)
    pos = np.arange(anchor_len, dtype=np.int32)
    bounds = np.zeros((shard.n_local, 2), dtype=np.int32)
    bounds[:] = (0, anchor_len)
    return src, pos, bounds


def global_split_order(plan):
    """(rank, local split) of every global split, in the single-GPU order:
    context blocks 0..n-1, then the tail."""
    order = []
    for s in plan:
        order += [(s.rank, j) for j in range(s.n_local)]
    q = plan[-1]
    order.append((q.rank, q.n_local))
    return order


def broadcast_query(q_buf, plan, group=None):
    """Every rank gets the query host's new tokens (Phase 2's broadcast)."""
    import torch.distributed as dist

    dist.broadcast(q_buf, src=plan[-1].rank, group=group)


def exchange_partials(send_o, send_lse, recv_o, recv_lse, slot_o, slot_lse, world, group=None):
    """All-gather of every rank's partial slot (the first slot_o / slot_lse
    floats of the send buffers) into rank-ordered recv buffers."""
    import torch.distributed as dist

    dist.all_gather_into_tensor(recv_o[:world * slot_o], send_o[:slot_o], group=group)
    dist.all_gather_into_tensor(recv_lse[:world * slot_lse], send_lse[:slot_lse], group=group)


def _view(t, shape):
    n = 1
    for d in shape:
        n *= d
    return t.view(-1)[:n].view(shape)


class ShardedStarLayer:
    """One attention layer's shard on this rank: its KV cache, Phase-1
    output and Phase-2 buffers (the library allocates nothing)."""

    def __init__(self, w: Workload, plan, rank, group=None, device="cuda"):
        self.w, self.plan, self.rank, self.group = w, plan, rank, group
        self.shard = s = plan[rank]
        B, Hq, Hkv, D = w.B, w.Hq, w.Hkv, w.D
        dev = torch.device(device)
        self.Tmax = max(w.Tq, 1)
        self.Lcap = s.rows + (w.Tq + w.Tdec if s.query_host else 0)
        self.S = max(p.nsplit for p in plan)  # split slots per rank in the exchange
        W = len(plan)
        self.k_cache = torch.empty((B, Hkv, self.Lcap, D), dtype=torch.bfloat16, device=dev)
        self.v_cache = torch.empty_like(self.k_cache)
        self.o = torch.empty((B, s.rows, Hq, D), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, Hq, s.rows), dtype=torch.float32, device=dev)
        if s.first_block == 0:
            self.ws1 = star.alloc_workspace(star.star_phase1_workspace_bytes(B, s.rows, Hq, D), dev)
            self.table = None
        else:
            a = w.anchor_len
            self.ws1 = star.alloc_workspace(
                star.star_phase1_ext_workspace_bytes(B, s.rows, Hq, Hkv, D, a), dev)
            self.table = tuple(torch.from_numpy(x).to(dev) for x in anchor_table(s, a))
        ws2 = max(star.star_phase2_workspace_bytes(B, t, Hq, Hkv, D, self.Lcap, w.block_len)
                  for t in (self.Tmax, 1))
        self.ws2 = star.alloc_workspace(ws2, dev)
        self.send_o = torch.empty(B * Hq * self.S * self.Tmax * D, dtype=torch.float32, device=dev)
        self.send_lse = torch.empty(B * Hq * self.S * self.Tmax, dtype=torch.float32, device=dev)
        self.recv_o = torch.empty(W * self.send_o.numel(), dtype=torch.float32, device=dev)
        self.recv_lse = torch.empty(W * self.send_lse.numel(), dtype=torch.float32, device=dev)
        self.q_buf = torch.empty((B, self.Tmax, Hq, D), dtype=torch.bfloat16, device=dev)
        self.o2 = torch.empty((B, self.Tmax, Hq, D), dtype=torch.bfloat16, device=dev)
        self.lse2 = torch.empty((B, Hq, self.Tmax), dtype=torch.float32, device=dev)

    # ---- Phase 1 --------------------------------------------------------------
    def encode(self, q, k, v, anchor_k=None, anchor_v=None):
        """q/k/v: this shard's context rows [B, rows, H, D] (pre-RoPE);
        anchor_k/v: the sequence's first anchor_len rows of k/v, needed by
        every shard without block 0."""
        w, s = self.w, self.shard
        if self.table is None:
            star.star_phase1_encode(q, k, v, self.o, self.k_cache, self.v_cache, w.block_len,
                                    w.anchor_len, w.theta, self.ws1, lse=self.lse)
        else:
            if anchor_k is None or anchor_v is None:
                raise ValueError("a shard without block 0 needs the anchor rows")
            src, pos, bounds = self.table
            star.star_phase1_encode_ext(q, k, v, self.o, self.k_cache, self.v_cache, w.block_len,
                                        w.theta, self.ws1, prefix_src=src, prefix_pos=pos,
                                        prefix_bounds=bounds, extra_k=anchor_k, extra_v=anchor_v,
                                        lse=self.lse, ctx_pos0=s.row0)
        return self.o

    # ---- Phase 2 --------------------------------------------------------------
    def local_partials(self, q, k, v, tail_len):
        """This rank's partials of T new tokens (q on every rank; k/v used by
        the query host only), written densely at the start of the send
        buffers. Returns (part_o [B, Hq, nsplit, T, D], part_lse [B, Hq,
        nsplit, T])."""
        w, s = self.w, self.shard
        B, T, Hq, D = q.shape
        po = _view(self.send_o, (B, Hq, s.nsplit, T, D))
        pl = _view(self.send_lse, (B, Hq, s.nsplit, T))
        q_pos0 = w.L + tail_len
        ns = star.star_phase2_partial_ext(
            q, k, v, self.k_cache, self.v_cache, s.rows, w.block_len,
            tail_len if s.query_host else 0, s.row0, q_pos0, s.query_host, po, pl, w.theta,
            self.ws2)
        if ns != s.nsplit:
            raise RuntimeError(f"rank {self.rank}: {ns} splits, planned {s.nsplit}")
        return po, pl

    def slot_sizes(self, T):
        """Floats per rank in the exchange of part_o and part_lse."""
        w = self.w
        return w.B * w.Hq * self.S * T * w.D, w.B * w.Hq * self.S * T

    def merge(self, T):
        """Exact merge of the gathered partials of every rank."""
        w = self.w
        o = _view(self.o2, (w.B, T, w.Hq, w.D))
        lse = _view(self.lse2, (w.B, w.Hq, T))
        star.star_lse_merge_ranks(self.recv_o, self.recv_lse, [p.nsplit for p in self.plan],
                                  self.S, o, lse)
        return o, lse

    def attend(self, q, k, v, tail_len):
        """One Phase-2 call across the ranks: broadcast q from the query
        host, local partials, all-gather, merge. Every rank returns the merged
        (o [B, T, Hq, D], lse [B, Hq, T])."""
        B, T, Hq, D = q.shape
        qb = _view(self.q_buf, (B, T, Hq, D))
        if self.shard.query_host:
            qb.copy_(q)
        broadcast_query(qb, self.plan, self.group)
        self.local_partials(qb, k, v, tail_len)
        n_o, n_l = self.slot_sizes(T)
        exchange_partials(self.send_o, self.send_lse, self.recv_o, self.recv_lse, n_o, n_l,
                          len(self.plan), self.group)
        return self.merge(T)
