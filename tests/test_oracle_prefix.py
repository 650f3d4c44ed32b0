"""Pins of the oracle's generalised Phase 1 (prefix variants).

The pages ablate the anchor (removed, position IDs changed, content
replaced; atlas.scime.ai summary, measured-effects table) and the Pulsar
follow-up replaces it with a 64-token sink plus chunks of earlier blocks at
their original positions (pith 2607.20457, "What carries the argument").
Checked against: the Star oracle when the prefix is the anchor, a dense-mask
brute force for arbitrary ranges, and the literal [explicit anchor || block]
concatenation for an anchor of given content and positions.
"""
import numpy as np
import pytest
import torch

from oracle import brute
from oracle import oracle as orc


def _inputs(L, Hq, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(1, L, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(1, L, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(1, L, Hkv, D, generator=g).to(torch.bfloat16)
    return q, k, v


def _all(L, Hq):
    hh, rr = np.meshgrid(np.arange(Hq), np.arange(L), indexing="ij")
    return np.zeros(hh.size, dtype=np.int64), hh.ravel(), rr.ravel()


def _rot(x, theta):
    return brute.rope_complex(x.double().numpy()[0], np.arange(x.shape[1]), theta)


@pytest.mark.parametrize("L,b,a", [(64, 16, 16), (50, 12, 5), (40, 10, 0)])
def test_anchor_prefix_equals_star(L, b, a):
    q, k, v = _inputs(L, 4, 2, 8, seed=L)
    n = -(-L // b)
    pre = np.zeros((n, 1, 2), dtype=np.int64)
    pre[1:, 0] = (0, a)
    qb, qh, qr = _all(L, 4)
    o, l, _ = orc.phase1_ext_rows(q, k, v, b, pre, 1e4, qb, qh, qr)
    so, sl, _ = orc.phase1_rows(q, k, v, b, a, 1e4, qb, qh, qr)
    np.testing.assert_array_equal(o, so)
    np.testing.assert_array_equal(l, sl)


@pytest.mark.parametrize("seed", range(6))
def test_arbitrary_prefix_ranges_match_dense_mask(seed):
    rng = np.random.default_rng(seed)
    L, b, Hq, Hkv, D = 72, 16, 4, 2, 8
    n = -(-L // b)
    R = 4
    pre = np.zeros((n, R, 2), dtype=np.int64)
    lists = [[] for _ in range(n)]
    for i in range(1, n):
        for j in range(R):
            if rng.random() < 0.7:
                s = int(rng.integers(0, i * b))
                e = int(rng.integers(s, i * b + 1))
                pre[i, j] = (s, e)
                lists[i].append((s, e))
    # overlapping ranges would count keys twice: keep them disjoint
    for i in range(1, n):
        seen = np.zeros(L, dtype=bool)
        for j in range(R):
            s, e = pre[i, j]
            if e > s and seen[s:e].any():
                pre[i, j] = (0, 0)
            elif e > s:
                seen[s:e] = True
        lists[i] = [tuple(x) for x in pre[i] if x[1] > x[0]]
    q, k, v = _inputs(L, Hq, Hkv, D, seed=100 + seed)
    qb, qh, qr = _all(L, Hq)
    o, l, _ = orc.phase1_ext_rows(q, k, v, b, pre, 1e4, qb, qh, qr, round_qk=False)
    M = brute.prefix_mask(L, b, lists)
    qr_, kr_ = _rot(q, 1e4), _rot(k, 1e4)
    vd = v.double().numpy()[0]
    for h in range(Hq):
        ro, rl = brute.masked_attention(qr_[:, h], kr_[:, h // 2], vd[:, h // 2], M)
        sel = qh == h
        np.testing.assert_allclose(o[sel], ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[sel], rl, rtol=0, atol=1e-12)


def test_pulsar_like_sink_and_summaries():
    # a 4-token sink from block 0 plus two 2-token chunks of every earlier block
    L, b = 64, 16
    n = L // b
    pre = np.zeros((n, 1 + 2 * (n - 1), 2), dtype=np.int64)
    lists = [[] for _ in range(n)]
    for i in range(1, n):
        rows = [(0, 4)] + [(j * b + 5, j * b + 7) for j in range(1, i)] + \
               [(j * b + 11, j * b + 13) for j in range(i)]
        for t, rg in enumerate(rows):
            pre[i, t] = rg
        lists[i] = rows
    q, k, v = _inputs(L, 2, 1, 8, seed=7)
    qb, qh, qr = _all(L, 2)
    o, l, nvis = orc.phase1_ext_rows(q, k, v, b, pre, 1e4, qb, qh, qr, round_qk=False)
    M = brute.prefix_mask(L, b, lists)
    assert (nvis[qh == 0] == M.sum(1)).all()
    ro, rl = brute.masked_attention(_rot(q, 1e4)[:, 0], _rot(k, 1e4)[:, 0], v.double().numpy()[0, :, 0], M)
    np.testing.assert_allclose(o[qh == 0], ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l[qh == 0], rl, rtol=0, atol=1e-12)


@pytest.mark.parametrize("La,pos_kind", [(8, "shifted"), (5, "random"), (16, "original")])
def test_explicit_anchor_matches_literal_concatenation(La, pos_kind):
    L, b, Hq, Hkv, D, theta = 48, 16, 4, 2, 8, 1e4
    q, k, v = _inputs(L, Hq, Hkv, D, seed=La)
    g = torch.Generator().manual_seed(99 + La)
    ak = torch.randn(1, La, Hkv, D, generator=g).to(torch.bfloat16)
    av = torch.randn(1, La, Hkv, D, generator=g).to(torch.bfloat16)
    if pos_kind == "shifted":
        apos = np.arange(La) + 1000
    elif pos_kind == "random":
        apos = np.random.default_rng(La).integers(0, 5000, size=La)
    else:
        apos = np.arange(La)
    n = L // b
    pre = np.zeros((n, 1, 2), dtype=np.int64)
    qb, qh, qr = _all(L, Hq)
    o, l, _ = orc.phase1_ext_rows(q, k, v, b, pre, theta, qb, qh, qr, anchor_k=ak, anchor_v=av,
                                  anchor_pos=apos, round_qk=False)
    ro, rl = brute.explicit_anchor_literal(q.double().numpy()[0], k.double().numpy()[0],
                                           v.double().numpy()[0], b, ak.double().numpy()[0],
                                           av.double().numpy()[0], apos, theta)
    for h in range(Hq):
        np.testing.assert_allclose(o[qh == h], ro[:, h], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[qh == h], rl[h], rtol=0, atol=1e-12)


def test_explicit_anchor_of_block_one_at_original_positions_is_star():
    L, b, a = 48, 16, 16
    q, k, v = _inputs(L, 2, 1, 8, seed=3)
    pre = np.zeros((L // b, 1, 2), dtype=np.int64)
    qb, qh, qr = _all(L, 2)
    o, l, _ = orc.phase1_ext_rows(q, k, v, b, pre, 1e4, qb, qh, qr, anchor_k=k[:, :a],
                                  anchor_v=v[:, :a], anchor_pos=np.arange(a))
    so, sl, _ = orc.phase1_rows(q, k, v, b, a, 1e4, qb, qh, qr)
    np.testing.assert_allclose(o, so, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l, sl, rtol=0, atol=1e-13)
