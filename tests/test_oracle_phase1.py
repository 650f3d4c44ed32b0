"""Pins of the oracle's Phase 1 (anchor-block blockwise-local causal encoding).

Checked against: full causal attention when one block covers the context
(c'_1 = c_1, pith 2WVXFXZ2 minor comment on Section 2.1); a dense-mask brute
force and the literal [anchor || block] concatenation of the augmented block
(pith 2WVXFXZ2 "What carries the argument"); closed forms (Q = 0 and
constant V); and the count of visible pairs.
"""
import itertools

import numpy as np
import pytest
import torch

from oracle import brute
from oracle import oracle as orc


def _inputs(L, Hq, Hkv, D, seed, q_scale=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(1, L, Hq, D, generator=g) * q_scale).to(torch.bfloat16)
    k = torch.randn(1, L, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(1, L, Hkv, D, generator=g).to(torch.bfloat16)
    return q, k, v


def _rot(x, theta):
    L = x.shape[1]
    return brute.rope_complex(x.double().numpy()[0], np.arange(L), theta)


@pytest.mark.parametrize("L,b,a", [(33, 33, 0), (33, 40, 0), (33, 64, 33), (50, 50, 7)])
def test_single_block_is_full_causal_attention(L, b, a):
    q, k, v = _inputs(L, 4, 2, 8, seed=L + b + a)
    o, lse = orc.phase1_full(q, k, v, b, a, 1e4, round_qk=False)
    ro, rl = brute.causal_full(_rot(q, 1e4), _rot(k, 1e4), v.double().numpy()[0])
    np.testing.assert_allclose(o[0], ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], rl, rtol=0, atol=1e-12)


_SHAPES = [(17, 1, 4), (40, 2, 8), (64, 4, 4), (64, 1, 8)]  # (L, g, D)
_BA = [(1, 0), (1, 1), (3, 0), (3, 2), (5, 5), (7, 3), (8, 8), (13, 1), (16, 0), (16, 16),
       (21, 10), (32, 32)]


@pytest.mark.parametrize("shape,ba", list(itertools.product(_SHAPES, _BA)))
def test_matches_dense_mask_brute_force(shape, ba):
    L, g, D = shape
    b, a = ba
    if b > L:
        pytest.skip("b > L is the single-block case")
    Hkv = 2
    q, k, v = _inputs(L, g * Hkv, Hkv, D, seed=1000 + L * 7 + b * 3 + a)
    o, lse = orc.phase1_full(q, k, v, b, a, 1e4, round_qk=False)
    ro, rl = brute.phase1_dense(_rot(q, 1e4), _rot(k, 1e4), v.double().numpy()[0], b, a)
    np.testing.assert_allclose(o[0], ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], rl, rtol=0, atol=1e-12)


@pytest.mark.parametrize("L,b,a,g", [(24, 8, 8, 1), (30, 7, 3, 2), (64, 16, 16, 4), (45, 10, 0, 2),
                                     (40, 12, 5, 1)])
def test_matches_literal_augmented_block(L, b, a, g):
    Hkv, D = 2, 8
    q, k, v = _inputs(L, g * Hkv, Hkv, D, seed=77 + L + b)
    o, lse = orc.phase1_full(q, k, v, b, a, 1e4, round_qk=False)
    ro, rl = brute.phase1_literal(q.double().numpy()[0], k.double().numpy()[0],
                                  v.double().numpy()[0], b, a, 1e4)
    np.testing.assert_allclose(o[0], ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], rl, rtol=0, atol=1e-12)


def test_peaked_softmax_and_sink_stress():
    L, b, a = 48, 12, 12
    q, k, v = _inputs(L, 4, 2, 8, seed=5, q_scale=8.0)
    k[0, 0] = (k[0, 0].float() * 6).to(torch.bfloat16)  # key 0 as a strong sink
    o, lse = orc.phase1_full(q, k, v, b, a, 1e4, round_qk=False)
    ro, rl = brute.phase1_dense(_rot(q, 1e4), _rot(k, 1e4), v.double().numpy()[0], b, a)
    np.testing.assert_allclose(o[0], ro, rtol=0, atol=1e-11)
    np.testing.assert_allclose(lse[0], rl, rtol=0, atol=1e-11)


@pytest.mark.parametrize("L,b,a", [(64, 16, 16), (50, 12, 5), (33, 8, 0)])
def test_zero_query_gives_mean_of_visible_values(L, b, a):
    q, k, v = _inputs(L, 2, 1, 8, seed=9)
    q.zero_()
    o, lse = orc.phase1_full(q, k, v, b, a, 1e4)
    M = brute.phase1_mask(L, b, a)
    vd = v.double().numpy()[0, :, 0]
    mean = (M.astype(np.float64) @ vd) / M.sum(1, keepdims=True)
    for h in range(2):
        np.testing.assert_allclose(o[0, :, h], mean, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0, h], np.log(M.sum(1)), rtol=0, atol=1e-13)


def test_constant_values_give_that_constant():
    L, b, a = 40, 10, 10
    q, k, v = _inputs(L, 2, 1, 8, seed=10)
    v[:] = 0.75
    o, _ = orc.phase1_full(q, k, v, b, a, 1e4)
    np.testing.assert_allclose(o, 0.75, rtol=0, atol=1e-13)


@pytest.mark.parametrize("L,b,a", [(64, 16, 16), (64, 16, 4), (96, 32, 0), (2048, 512, 512)])
def test_visible_pair_count(L, b, a):
    n = L // b
    q, k, v = _inputs(L, 1, 1, 4, seed=11)
    rows = np.arange(L)
    _, _, nvis = orc.phase1_rows(q, k, v, b, a, 1e4, np.zeros(L), np.zeros(L), rows)
    assert nvis.sum() == n * b * (b + 1) // 2 + (n - 1) * a * b


def test_ranges_match_dense_mask():
    for L, b, a in [(37, 5, 3), (64, 16, 16), (20, 20, 20), (31, 4, 0)]:
        blk, rng = orc.phase1_ranges(L, b, a)
        M = brute.phase1_mask(L, b, a)
        for r in range(L):
            assert blk[r] == r // b
            vis = np.zeros(L, dtype=bool)
            vis[rng[r, 0]:rng[r, 1]] = True
            vis[rng[r, 2]:rng[r, 3]] = True
            np.testing.assert_array_equal(vis, M[r])


def test_rounded_qk_mode_equals_brute_on_rounded_inputs():
    L, b, a, theta = 40, 10, 10, 1e4
    q, k, v = _inputs(L, 4, 2, 8, seed=12)
    o, lse = orc.phase1_full(q, k, v, b, a, theta, round_qk=True)
    qr = brute.round_bf16_np(_rot(q, theta))
    kr = brute.round_bf16_np(_rot(k, theta))
    ro, rl = brute.phase1_dense(qr, kr, v.double().numpy()[0], b, a)
    # the two rotations may land on opposite sides of a bf16 rounding boundary
    # only if they differ by >1e-15 relative; with ~2000 values that never
    # happens here, so agreement is to fp64 rounding of the attention itself
    np.testing.assert_allclose(o[0], ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], rl, rtol=0, atol=1e-12)


def _edge_rows(L, b):
    """Rows at block starts and ends, 128-row tile edges, and a few inside."""
    rows = set()
    for s in range(0, L, b):
        for r in (s, s + 1, s + b - 1, s + b - 2):
            if 0 <= r < L:
                rows.add(r)
        for t in range(s, min(s + b, L), 128):
            for r in (t - 1, t, t + 127):
                if s <= r < min(s + b, L):
                    rows.add(r)
    rows.add(L - 1)
    return sorted(rows)


@pytest.mark.parametrize("B,L,b,a,g,Hkv", [(2, 300, 128, 128, 1, 2), (2, 1000, 300, 200, 4, 2),
                                           (3, 520, 256, 100, 8, 1), (2, 640, 640, 640, 4, 1),
                                           (2, 777, 129, 0, 8, 2)])
def test_selected_rows_equal_full_tensor_rows(B, L, b, a, g, Hkv):
    """phase1_rows_selected (queries passed one by one, as the full-size
    checks do) gives exactly the bits of phase1_rows on the whole Q tensor,
    for random (batch, head, row) picks and rows at block and tile edges."""
    Hq, D, theta = g * Hkv, 16, 5e5
    gen = torch.Generator().manual_seed(B * 1000 + L + b + a + g)
    q = torch.randn(B, L, Hq, D, generator=gen).to(torch.bfloat16)
    k = torch.randn(B, L, Hkv, D, generator=gen).to(torch.bfloat16)
    v = torch.randn(B, L, Hkv, D, generator=gen).to(torch.bfloat16)
    rng = np.random.default_rng(L + b)
    edge = np.array(_edge_rows(L, b))
    nr = 60
    rows = np.concatenate([edge, rng.integers(0, L, size=nr)])
    qb = rng.integers(0, B, size=rows.size)
    qh = rng.integers(0, Hq, size=rows.size)
    perm = rng.permutation(rows.size)  # the selection's order is arbitrary
    rows, qb, qh = rows[perm], qb[perm], qh[perm]
    q_sel = q[torch.as_tensor(qb), torch.as_tensor(rows), torch.as_tensor(qh)]  # [nq, D]
    for round_qk in (True, False):
        o_ref, l_ref, n_ref = orc.phase1_rows(q, k, v, b, a, theta, qb, qh, rows, round_qk)
        o, lse, nvis = orc.phase1_rows_selected(q_sel, k, v, b, a, theta, qb, qh, rows, Hq,
                                                round_qk)
        np.testing.assert_array_equal(o, o_ref)
        np.testing.assert_array_equal(lse, l_ref)
        np.testing.assert_array_equal(nvis, n_ref)


@pytest.mark.parametrize("L,b,a,g", [(48, 12, 12, 1), (50, 16, 5, 4), (40, 40, 40, 8),
                                     (45, 10, 0, 2)])
def test_selected_rows_match_dense_mask_brute_force(L, b, a, g):
    """phase1_rows_selected against the dense-mask brute force directly, on
    every row of two sequences, heads of every GQA group, rows given in
    reverse order."""
    B, Hkv, D, theta = 2, 2, 8, 1e4
    Hq = g * Hkv
    gen = torch.Generator().manual_seed(400 + L + b + a + g)
    q = torch.randn(B, L, Hq, D, generator=gen).to(torch.bfloat16)
    k = torch.randn(B, L, Hkv, D, generator=gen).to(torch.bfloat16)
    v = torch.randn(B, L, Hkv, D, generator=gen).to(torch.bfloat16)
    bb, hh, rr = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(L)[::-1], indexing="ij")
    qb, qh, qr = bb.ravel(), hh.ravel(), rr.ravel()
    q_sel = q[torch.as_tensor(qb), torch.as_tensor(qr), torch.as_tensor(qh)]
    o, lse, nvis = orc.phase1_rows_selected(q_sel, k, v, b, a, theta, qb, qh, qr, Hq,
                                            round_qk=False)
    M = brute.phase1_mask(L, b, a)
    for bi in range(B):
        qrot = brute.rope_complex(q[bi].double().numpy(), np.arange(L), theta)
        krot = brute.rope_complex(k[bi].double().numpy(), np.arange(L), theta)
        ro, rl = brute.phase1_dense(qrot, krot, v[bi].double().numpy(), b, a)
        sel = qb == bi
        np.testing.assert_allclose(o[sel], ro[qr[sel], qh[sel]], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[sel], rl[qh[sel], qr[sel]], rtol=0, atol=1e-12)
        np.testing.assert_array_equal(nvis[sel], M.sum(1)[qr[sel]])
