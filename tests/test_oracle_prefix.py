"""Pins of the oracle's generalised Phase 1 (gathered prefix table).

The pages ablate the anchor (removed, position IDs changed, content
replaced; atlas.scime.ai summary, measured-effects table) and the Pulsar
follow-up replaces it with a 64-token sink plus chunks of earlier blocks at
their original global positions, block i seeing [sink || Sigma_0 || ... ||
Sigma_{i-1}] (pith 2607.20457, "What carries the argument"). All of them are
one prefix table (rows of the context or given rows, each rotated at a given
position) of which block i sees a slice.
Checked against: the Star oracle when the table is the anchor, a dense-mask
brute force when the table holds context rows at their own positions, and
the literal [prefix rows || block] concatenation for given content and
positions.
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


def _table(per_block):
    """Concatenate per-block lists of context ranges into (src, bounds)."""
    src, bounds = [], []
    for rows in per_block:
        gs = len(src)
        for s, e in rows:
            src.extend(range(s, e))
        bounds.append((gs, len(src)))
    return np.asarray(src, dtype=np.int64), np.asarray(bounds, dtype=np.int64)


@pytest.mark.parametrize("L,b,a", [(64, 16, 16), (50, 12, 5), (40, 10, 0)])
def test_anchor_table_equals_star(L, b, a):
    q, k, v = _inputs(L, 4, 2, 8, seed=L)
    n = -(-L // b)
    bounds = np.zeros((n, 2), dtype=np.int64)
    bounds[1:] = (0, a)
    qb, qh, qr = _all(L, 4)
    o, l, _ = orc.phase1_gather_rows(q, k, v, b, np.arange(a), np.arange(a), bounds, 1e4, qb, qh, qr)
    so, sl, _ = orc.phase1_rows(q, k, v, b, a, 1e4, qb, qh, qr)
    np.testing.assert_array_equal(o, so)
    np.testing.assert_array_equal(l, sl)


@pytest.mark.parametrize("seed", range(6))
def test_context_row_tables_match_dense_mask(seed):
    rng = np.random.default_rng(seed)
    L, b, Hq, Hkv, D = 72, 16, 4, 2, 8
    n = -(-L // b)
    lists = []
    for i in range(n):
        seen = np.zeros(L, dtype=bool)
        rows = []
        for _ in range(4):
            if i == 0 or rng.random() >= 0.7:
                continue
            s = int(rng.integers(0, i * b))
            e = int(rng.integers(s, i * b + 1))
            if e > s and not seen[s:e].any():  # a row listed twice would count twice
                seen[s:e] = True
                rows.append((s, e))
        lists.append(rows)
    src, bounds = _table(lists)
    q, k, v = _inputs(L, Hq, Hkv, D, seed=100 + seed)
    qb, qh, qr = _all(L, Hq)
    o, l, nvis = orc.phase1_gather_rows(q, k, v, b, src, src, bounds, 1e4, qb, qh, qr,
                                        round_qk=False)
    M = brute.prefix_mask(L, b, lists)
    qr_, kr_ = _rot(q, 1e4), _rot(k, 1e4)
    vd = v.double().numpy()[0]
    for h in range(Hq):
        ro, rl = brute.masked_attention(qr_[:, h], kr_[:, h // 2], vd[:, h // 2], M)
        sel = qh == h
        assert (nvis[sel] == M.sum(1)).all()
        np.testing.assert_allclose(o[sel], ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[sel], rl, rtol=0, atol=1e-12)


def test_pulsar_nested_table_matches_dense_mask():
    # a 4-token sink from block 0 plus, per block, two 2-token chunks; block i
    # sees the sink and the chunks of blocks 0..i-1 (a prefix of the table)
    L, b = 64, 16
    n = L // b
    sink = [(0, 4)]
    chunks = [[(j * b + 5, j * b + 7), (j * b + 11, j * b + 13)] for j in range(n)]
    src = list(range(0, 4))
    bounds = [(0, 0)]
    for i in range(1, n):
        for s, e in chunks[i - 1]:
            src.extend(range(s, e))
        bounds.append((0, len(src)))
    src = np.asarray(src)
    lists = [[]] + [sink + sum(chunks[:i], []) for i in range(1, n)]
    q, k, v = _inputs(L, 2, 1, 8, seed=7)
    qb, qh, qr = _all(L, 2)
    o, l, nvis = orc.phase1_gather_rows(q, k, v, b, src, src, np.asarray(bounds), 1e4, qb, qh, qr,
                                        round_qk=False)
    M = brute.prefix_mask(L, b, lists)
    assert (nvis[qh == 0] == M.sum(1)).all()
    ro, rl = brute.masked_attention(_rot(q, 1e4)[:, 0], _rot(k, 1e4)[:, 0], v.double().numpy()[0, :, 0], M)
    np.testing.assert_allclose(o[qh == 0], ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l[qh == 0], rl, rtol=0, atol=1e-12)


@pytest.mark.parametrize("La,pos_kind", [(8, "shifted"), (5, "random"), (16, "original")])
def test_given_rows_match_literal_concatenation(La, pos_kind):
    L, b, Hq, Hkv, D, theta = 48, 16, 4, 2, 8, 1e4
    q, k, v = _inputs(L, Hq, Hkv, D, seed=La)
    g = torch.Generator().manual_seed(99 + La)
    xk = torch.randn(1, La, Hkv, D, generator=g).to(torch.bfloat16)
    xv = torch.randn(1, La, Hkv, D, generator=g).to(torch.bfloat16)
    if pos_kind == "shifted":
        pos = np.arange(La) + 1000
    elif pos_kind == "random":
        pos = np.random.default_rng(La).integers(0, 5000, size=La)
    else:
        pos = np.arange(La)
    n = L // b
    bounds = np.zeros((n, 2), dtype=np.int64)
    bounds[1:] = (0, La)
    qb, qh, qr = _all(L, Hq)
    o, l, _ = orc.phase1_gather_rows(q, k, v, b, -1 - np.arange(La), pos, bounds, theta, qb, qh, qr,
                                     extra_k=xk, extra_v=xv, round_qk=False)
    ro, rl = brute.gathered_prefix_literal(q.double().numpy()[0], k.double().numpy()[0],
                                           v.double().numpy()[0], b, xk.double().numpy()[0],
                                           xv.double().numpy()[0], pos, bounds, theta)
    for h in range(Hq):
        np.testing.assert_allclose(o[qh == h], ro[:, h], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[qh == h], rl[h], rtol=0, atol=1e-12)


def test_mixed_table_with_block_zero_prefix_and_repeats_matches_literal():
    # given rows and context rows mixed, a row listed twice, a row of the
    # block's own future at a moved position, and a prefix for block 0 too
    L, b, Hq, Hkv, D, theta = 40, 10, 2, 1, 8, 1e4
    q, k, v = _inputs(L, Hq, Hkv, D, seed=5)
    g = torch.Generator().manual_seed(5)
    xk = torch.randn(1, 3, Hkv, D, generator=g).to(torch.bfloat16)
    xv = torch.randn(1, 3, Hkv, D, generator=g).to(torch.bfloat16)
    src = np.array([-1, -2, 3, 3, 17, -3, 0, 25, 9])
    pos = np.array([-5, 7, 3, 3, 100, 2, 0, 25, 9000])
    bounds = np.array([(0, 2), (1, 6), (4, 9), (2, 2)])
    qb, qh, qr = _all(L, Hq)
    o, l, nvis = orc.phase1_gather_rows(q, k, v, b, src, pos, bounds, theta, qb, qh, qr,
                                        extra_k=xk, extra_v=xv, round_qk=False)
    kd, vd = k.double().numpy()[0], v.double().numpy()[0]
    xkd, xvd = xk.double().numpy()[0], xv.double().numpy()[0]
    pk = np.stack([kd[s] if s >= 0 else xkd[-1 - s] for s in src])
    pv = np.stack([vd[s] if s >= 0 else xvd[-1 - s] for s in src])
    ro, rl = brute.gathered_prefix_literal(q.double().numpy()[0], kd, vd, b, pk, pv, pos, bounds,
                                           theta)
    want = np.array([bounds[r // b][1] - bounds[r // b][0] + r % b + 1 for r in range(L)])
    assert (nvis[qh == 0] == want).all()
    for h in range(Hq):
        np.testing.assert_allclose(o[qh == h], ro[:, h], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[qh == h], rl[h], rtol=0, atol=1e-12)


def test_given_copy_of_block_one_at_original_positions_is_star():
    L, b, a = 48, 16, 16
    q, k, v = _inputs(L, 2, 1, 8, seed=3)
    bounds = np.zeros((L // b, 2), dtype=np.int64)
    bounds[1:] = (0, a)
    qb, qh, qr = _all(L, 2)
    o, l, _ = orc.phase1_gather_rows(q, k, v, b, -1 - np.arange(a), np.arange(a), bounds, 1e4,
                                     qb, qh, qr, extra_k=k[:, :a], extra_v=v[:, :a])
    so, sl, _ = orc.phase1_rows(q, k, v, b, a, 1e4, qb, qh, qr)
    np.testing.assert_allclose(o, so, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l, sl, rtol=0, atol=1e-13)
