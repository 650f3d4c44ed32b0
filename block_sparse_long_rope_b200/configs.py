"""The five single-layer workloads the hot path is measured and checked on.

Shapes are Llama-3.1 attention layers (8B: 32 query / 8 KV heads, 70B: 64 /
8, head_dim 128) plus a tiny GQA case; block size b and anchor size a follow
the pages' setting (b = L/4 for 16K-128K, larger fixed blocks beyond; anchor
size = block size) [pith 2WVXFXZ2, "Assumptions & free parameters"].
"""
from dataclasses import dataclass, field
from typing import List


@dataclass(frozen=True)
class Workload:
    index: int            # seed namespace (see inputs.seed_for)
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    theta: float
    L: int
    block_len: int
    anchor_len: int
    Tq: int               # Phase-2 query chunk tokens
    Tdec: int             # Phase-2 single-token decode steps

    @property
    def n_blocks(self) -> int:
        return -(-self.L // self.block_len)

    @property
    def Lcap(self) -> int:
        return self.L + self.Tq + self.Tdec

    def phase1_pairs_per_head(self) -> int:
        """Unmasked (query, key) pairs of Phase 1 for one (sequence, head)."""
        b, a, n, L = self.block_len, self.anchor_len, self.n_blocks, self.L
        total = 0
        for i in range(n):
            lo, hi = i * b, min((i + 1) * b, L)
            m = hi - lo
            total += m * (m + 1) // 2
            if i > 0:
                total += m * a
        return total

    def phase1_flops(self) -> float:
        """2 (QK^T) + 2 (PV) flops per head-dim element of each unmasked pair."""
        return 4.0 * self.D * self.Hq * self.B * self.phase1_pairs_per_head()

    def decode_kv_bytes(self, tail_len: int) -> float:
        """K+V cache bytes one decode step must read (bf16)."""
        return 2.0 * (self.L + tail_len + 1) * self.Hkv * self.D * 2 * self.B


def _w(**kw) -> Workload:
    return Workload(**kw)


WORKLOADS: List[Workload] = [
    _w(index=0, name="tiny-gqa-2k", B=1, Hq=4, Hkv=1, D=64, theta=1.0e4, L=2048, block_len=512,
       anchor_len=512, Tq=16, Tdec=8),
    _w(index=1, name="llama8b-16k", B=1, Hq=32, Hkv=8, D=128, theta=5.0e5, L=16384,
       block_len=4096, anchor_len=4096, Tq=128, Tdec=64),
    _w(index=2, name="llama8b-64k-b4k", B=1, Hq=32, Hkv=8, D=128, theta=5.0e5, L=65536,
       block_len=4096, anchor_len=4096, Tq=128, Tdec=128),
    _w(index=2, name="llama8b-64k-b16k", B=1, Hq=32, Hkv=8, D=128, theta=5.0e5, L=65536,
       block_len=16384, anchor_len=16384, Tq=128, Tdec=128),
    _w(index=2, name="llama8b-64k-b4k-batch4", B=4, Hq=32, Hkv=8, D=128, theta=5.0e5, L=65536,
       block_len=4096, anchor_len=4096, Tq=128, Tdec=128),
    _w(index=2, name="llama8b-64k-b16k-batch4", B=4, Hq=32, Hkv=8, D=128, theta=5.0e5, L=65536,
       block_len=16384, anchor_len=16384, Tq=128, Tdec=128),
    _w(index=3, name="llama70b-128k", B=1, Hq=64, Hkv=8, D=128, theta=5.0e5, L=131072,
       block_len=32768, anchor_len=32768, Tq=256, Tdec=128),
    _w(index=4, name="llama8b-1m", B=1, Hq=32, Hkv=8, D=128, theta=5.0e5, L=1048576,
       block_len=131072, anchor_len=131072, Tq=64, Tdec=32),
]

BY_NAME = {w.name: w for w in WORKLOADS}
