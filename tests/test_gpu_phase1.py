"""GPU parity of Phase 1 (star_phase1_encode) against the fp64 oracle, element
by element on shapes that span several 128-row tiles and ragged tails, plus
the degenerate cases: no anchor, anchor shorter than the block, one block
covering the context (full causal), one-token blocks, GQA group sizes 1/2/4/8
and both head dims."""
import numpy as np
import pytest
import torch

from block_sparse_long_rope_b200 import build as star_build
from block_sparse_long_rope_b200 import star
from oracle import oracle as orc

from gpu_util import TOL_LSE, TOL_O, max_abs, rand_bf16, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    star_build.build()
    torch.cuda.init()


def encode(q, k, v, b, a, theta, Lcap=None, with_lse=True):
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    Lcap = Lcap or L
    dev = q.device
    o = torch.empty_like(q)
    kc = torch.full((B, Hkv, Lcap, D), float("nan"), dtype=torch.bfloat16, device=dev)
    vc = torch.full((B, Hkv, Lcap, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev) if with_lse else None
    ws = star.alloc_workspace(star.star_phase1_workspace_bytes(B, L, Hq, D), dev)
    ws.fill_(0xFF)  # poison: reads of unwritten workspace show up as NaN
    ws[:256].zero_()
    star.star_phase1_encode(q, k, v, o, kc, vc, b, a, theta, ws, lse=lse)
    star.star_device_status(ws)
    return o, lse, kc, vc


# (B, L, Hq, Hkv, D, block_len, anchor_len, theta)
SHAPES = [
    (1, 2048, 4, 1, 64, 512, 512, 1e4),      # the tiny GQA configuration
    (2, 1000, 4, 2, 64, 300, 100, 1e4),      # ragged blocks and tiles, anchor < block
    (1, 777, 3, 3, 128, 256, 200, 5e5),      # g = 1 (one head per CTA)
    (1, 640, 2, 1, 128, 128, 0, 5e5),        # no anchor (the pages' ablation)
    (1, 500, 2, 2, 128, 1024, 0, 5e5),       # one block: full causal attention
    (1, 1536, 8, 2, 128, 512, 128, 5e5),     # anchor of a quarter block
    (1, 500, 4, 2, 64, 64, 64, 1e4),         # blocks shorter than a tile
    (1, 100, 2, 1, 128, 1, 1, 5e5),          # one-token blocks
    (1, 1300, 16, 2, 128, 650, 650, 5e5),    # g = 8
]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"L{s[1]}b{s[5]}a{s[6]}g{s[2]//s[3]}D{s[4]}" for s in SHAPES])
def test_phase1_matches_oracle_everywhere(shape):
    B, L, Hq, Hkv, D, b, a, theta = shape
    q = rand_bf16((B, L, Hq, D), seed=L + 1)
    k = rand_bf16((B, L, Hkv, D), seed=L + 2)
    v = rand_bf16((B, L, Hkv, D), seed=L + 3)
    o, lse, kc, vc = encode(q, k, v, b, a, theta, Lcap=L + 37)
    torch.cuda.synchronize()
    ro, rl = orc.phase1_full(q.cpu(), k.cpu(), v.cpu(), b, a, theta)
    assert max_abs(to64(o), ro) <= TOL_O
    assert max_abs(to64(lse), rl) <= TOL_LSE
    # cache rows [0, L): K rotated at its position, V copied bit for bit
    kref = orc.rope(k.cpu(), np.arange(L), theta, round_out=True)  # [B, L, Hkv, D]
    kgot = to64(kc[:, :, :L]).transpose(0, 2, 1, 3)
    np.testing.assert_array_equal(kgot, kref)  # correctly rounded: bit-exact
    assert torch.equal(vc[:, :, :L].permute(0, 2, 1, 3).cpu(), v.cpu())
    assert torch.isnan(kc[:, :, L:].float()).all()  # rows past L untouched


def test_phase1_zero_query_counts_visible_keys():
    # with Q = 0 every visible key scores 0, so exp(LSE) is the number of
    # visible keys exactly: the behavioural check of the kernels' masks
    B, L, Hq, Hkv, D, b, a = 1, 1100, 4, 2, 128, 384, 200
    q = torch.zeros((B, L, Hq, D), dtype=torch.bfloat16, device="cuda")
    k = rand_bf16((B, L, Hkv, D), seed=1)
    v = rand_bf16((B, L, Hkv, D), seed=2)
    _, lse, _, _ = encode(q, k, v, b, a, 5e5)
    torch.cuda.synchronize()
    counts = np.rint(np.exp(to64(lse)))
    _, rng = orc.phase1_ranges(L, b, a)
    want = (rng[:, 1] - rng[:, 0]) + (rng[:, 3] - rng[:, 2])
    for h in range(Hq):
        np.testing.assert_array_equal(counts[0, h], want)


def test_phase1_peaked_softmax_and_sink():
    B, L, Hq, Hkv, D, b, a, theta = 1, 1024, 4, 2, 128, 256, 256, 5e5
    q = rand_bf16((B, L, Hq, D), seed=11, scale=8.0)
    k = rand_bf16((B, L, Hkv, D), seed=12)
    k[:, 0] *= 6  # key 0 as a strong attention sink
    v = rand_bf16((B, L, Hkv, D), seed=13)
    o, lse, _, _ = encode(q, k, v, b, a, theta)
    torch.cuda.synchronize()
    ro, rl = orc.phase1_full(q.cpu(), k.cpu(), v.cpu(), b, a, theta)
    assert max_abs(to64(o), ro) <= TOL_O
    assert max_abs(to64(lse), rl) <= TOL_LSE


def test_phase1_without_lse_and_repeatable():
    B, L, Hq, Hkv, D, b, a, theta = 1, 700, 4, 1, 64, 256, 256, 1e4
    q = rand_bf16((B, L, Hq, D), seed=21)
    k = rand_bf16((B, L, Hkv, D), seed=22)
    v = rand_bf16((B, L, Hkv, D), seed=23)
    o1, _, _, _ = encode(q, k, v, b, a, theta, with_lse=False)
    o2, _, _, _ = encode(q, k, v, b, a, theta)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)  # deterministic, LSE output optional
