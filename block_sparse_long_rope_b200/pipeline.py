"""One Star Attention layer through the C ABI: Phase 1 context encoding, a
Phase-2 query chunk, then single-token decode steps, each Phase-2 call
followed by the exact LSE merge [pith 2WVXFXZ2, abstract: "In the first
phase, the context is processed using blockwise-local attention ... In the
second phase, query and response tokens attend to all prior cached tokens"].

All buffers are allocated once here (the library allocates nothing) and
reused across steps; every call is enqueued on the current CUDA stream.
"""
from dataclasses import dataclass

import torch

from . import star
from .configs import Workload


@dataclass
class LayerBuffers:
    k_cache: torch.Tensor   # [B, Hkv, Lcap, D] bf16
    v_cache: torch.Tensor
    o: torch.Tensor         # [B, L, Hq, D] bf16
    lse: torch.Tensor       # [B, Hq, L] fp32
    ws1: torch.Tensor       # Phase-1 workspace
    ws2: torch.Tensor       # Phase-2 workspace (sized for the largest T)
    part_o: torch.Tensor    # [B, Hq, n+1, Tmax, D] fp32
    part_lse: torch.Tensor  # [B, Hq, n+1, Tmax]
    o2: torch.Tensor        # [B, Tmax, Hq, D] bf16 merged Phase-2 output
    lse2: torch.Tensor      # [B, Hq, Tmax]


class StarLayer:
    """Holds the caller-owned buffers of one attention layer of workload `w`."""

    def __init__(self, w: Workload, device="cuda"):
        self.w = w
        B, Hq, Hkv, D = w.B, w.Hq, w.Hkv, w.D
        n = w.n_blocks
        Tmax = max(w.Tq, 1)
        dev = torch.device(device)
        ws2 = max(star.star_phase2_workspace_bytes(B, t, Hq, Hkv, D, w.Lcap, w.block_len)
                  for t in (Tmax, 1))
        self.buf = LayerBuffers(
            k_cache=torch.empty((B, Hkv, w.Lcap, D), dtype=torch.bfloat16, device=dev),
            v_cache=torch.empty((B, Hkv, w.Lcap, D), dtype=torch.bfloat16, device=dev),
            o=torch.empty((B, w.L, Hq, D), dtype=torch.bfloat16, device=dev),
            lse=torch.empty((B, Hq, w.L), dtype=torch.float32, device=dev),
            ws1=star.alloc_workspace(star.star_phase1_workspace_bytes(B, w.L, Hq, D), dev),
            ws2=star.alloc_workspace(ws2, dev),
            part_o=torch.empty((B, Hq, n + 1, Tmax, D), dtype=torch.float32, device=dev),
            part_lse=torch.empty((B, Hq, n + 1, Tmax), dtype=torch.float32, device=dev),
            o2=torch.empty((B, Tmax, Hq, D), dtype=torch.bfloat16, device=dev),
            lse2=torch.empty((B, Hq, Tmax), dtype=torch.float32, device=dev),
        )

        self.prefix = None

    def set_prefix(self, src, pos, bounds, extra_k=None, extra_v=None):
        """Replace the Star anchor by a gathered prefix table (see prefix.py):
        later encode calls run star_phase1_encode_ext with it. None restores
        the anchor."""
        if src is None:
            self.prefix = None
            return
        w, dev = self.w, self.buf.o.device
        t = [torch.as_tensor(x, dtype=torch.int32).contiguous().to(dev) for x in (src, pos, bounds)]
        if t[2].shape != (w.n_blocks, 2):
            raise ValueError(f"bounds must be [{w.n_blocks}, 2]")
        G = t[0].numel()
        ws = star.alloc_workspace(
            star.star_phase1_ext_workspace_bytes(w.B, w.L, w.Hq, w.Hkv, w.D, G), dev)
        self.prefix = (t[0], t[1], t[2], extra_k, extra_v, ws)

    def encode(self, q, k, v, with_lse=True):
        b = self.buf
        lse = b.lse if with_lse else None
        if self.prefix is None:
            star.star_phase1_encode(q, k, v, b.o, b.k_cache, b.v_cache, self.w.block_len,
                                    self.w.anchor_len, self.w.theta, b.ws1, lse=lse)
        else:
            src, pos, bounds, xk, xv, ws = self.prefix
            star.star_phase1_encode_ext(q, k, v, b.o, b.k_cache, b.v_cache, self.w.block_len,
                                        self.w.theta, ws, prefix_src=src, prefix_pos=pos,
                                        prefix_bounds=bounds, extra_k=xk, extra_v=xv, lse=lse)
        return b.o

    @property
    def ws_phase1(self):
        return self.buf.ws1 if self.prefix is None else self.prefix[5]

    def partial(self, q, k, v, tail_len):
        """Phase-2 partials of T = q.shape[1] new tokens; returns contiguous views
        (part_o[B,Hq,n+1,T,D], part_lse[B,Hq,n+1,T]) of the layer's buffers."""
        b = self.buf
        B, T, Hq, D = q.shape
        S = b.part_o.shape[2]
        po = _prefix_view(b.part_o, (B, Hq, S, T, D))
        pl = _prefix_view(b.part_lse, (B, Hq, S, T))
        star.star_phase2_partial(q, k, v, b.k_cache, b.v_cache, self.w.L, self.w.block_len,
                                 tail_len, po, pl, self.w.theta, b.ws2)
        return po, pl

    def attend(self, q, k, v, tail_len):
        """Partials and their exact merge in one call (star_phase2_attend):
        returns (o[B,T,Hq,D] bf16, lse[B,Hq,T]) views of the layer's buffers."""
        b = self.buf
        B, T, Hq, D = q.shape
        S = b.part_o.shape[2]
        po = _prefix_view(b.part_o, (B, Hq, S, T, D))
        pl = _prefix_view(b.part_lse, (B, Hq, S, T))
        o = _prefix_view(b.o2, (B, T, Hq, D))
        lse = _prefix_view(b.lse2, (B, Hq, T))
        star.star_phase2_attend(q, k, v, b.k_cache, b.v_cache, self.w.L, self.w.block_len,
                                tail_len, po, pl, o, self.w.theta, b.ws2, lse=lse)
        return o, lse

    def attend_unfused(self, q, k, v, tail_len):
        """star_phase2_partial then star_lse_merge (two calls)."""
        po, pl = self.partial(q, k, v, tail_len)
        B, Hq, S, T, D = po.shape
        o = _prefix_view(self.buf.o2, (B, T, Hq, D))
        lse = _prefix_view(self.buf.lse2, (B, Hq, T))
        star.star_lse_merge(po, pl, o, lse)
        return o, lse

    def step(self, ctx, calls):
        """One full pass of the hot path: Phase 1 over the context, then the
        Phase-2 calls in order (the Tq-token query chunk, then Tdec
        single-token decode steps). ctx = (q, k, v); calls = list of
        (q, k, v, tail_len) with contiguous inputs (see phase2_calls).
        Returns the last merged output (o, lse)."""
        q, k, v = ctx
        self.encode(q, k, v)
        out = None
        for (q2, k2, v2, tail) in calls:
            out = self.attend(q2, k2, v2, tail)
        return out


def _prefix_view(t, shape):
    n = 1
    for d in shape:
        n *= d
    return t.view(-1)[:n].view(shape)


def phase2_calls(w: Workload, q2, k2, v2):
    """Split the Tq + Tdec Phase-2 tokens ([B, Tq+Tdec, H, D]) into the
    contiguous per-call inputs: one query chunk of Tq tokens, then Tdec
    single tokens, each with the tail length before it."""
    calls = []
    if w.Tq > 0:
        calls.append((q2[:, : w.Tq].contiguous(), k2[:, : w.Tq].contiguous(),
                      v2[:, : w.Tq].contiguous(), 0))
    for s in range(w.Tdec):
        t = w.Tq + s
        calls.append((q2[:, t:t + 1].contiguous(), k2[:, t:t + 1].contiguous(),
                      v2[:, t:t + 1].contiguous(), t))
    return calls
