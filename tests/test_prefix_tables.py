"""Host-side prefix-table builders (block_sparse_long_rope_b200.prefix),
checked against the pages' layouts and, through the oracle, against a dense
mask of the same visible sets."""
import numpy as np
import pytest
import torch

from block_sparse_long_rope_b200 import prefix as pfx
from oracle import brute
from oracle import oracle as orc


def test_star_table_pairs_match_the_star_count():
    # n*b(b+1)/2 + (n-1)*a*b visible pairs when b divides L
    for L, b, a in ((16384, 4096, 4096), (1024, 256, 100), (1024, 256, 0)):
        src, pos, bounds = pfx.star_table(L, b, a)
        n = L // b
        assert pfx.prefix_pairs(L, b, bounds) == n * b * (b + 1) // 2 + (n - 1) * a * b
        assert (src == np.arange(a)).all() and (pos == src).all()
        assert tuple(bounds[0]) == (0, 0)


def test_pulsar_table_layout():
    L, b = 16384, 4096
    chunks = pfx.draw_chunks(L, b, seed=3)
    assert len(chunks) == 3 and all(c.size == 16 for c in chunks)  # 12.5% of 4096 / 32
    assert chunks[0].min() >= 2                                     # outside the 64-token sink
    src, pos, bounds = pfx.pulsar_table(L, b, chunks)
    assert (pos == src).all()                                       # original positions
    assert (src[:64] == np.arange(64)).all()
    for i in range(1, 4):
        assert tuple(bounds[i]) == (0, 64 + 512 * i)                # nested: sink + Sigma_<i
        seen = src[bounds[i][0]:bounds[i][1]]
        assert (seen < i * b).all()                                 # only earlier blocks
        assert np.unique(seen).size == seen.size
    # the block-wise order: Sigma_j lies inside block j, ascending
    for j in range(3):
        part = src[64 + 512 * j:64 + 512 * (j + 1)]
        assert (part // b == j).all() and (np.diff(part) > 0).all()
    # Phase-1 pairs: the pages' cost model counts keys per host; Pulsar's are
    # a small part of Star's here
    star_pairs = pfx.prefix_pairs(L, b, pfx.star_table(L, b, b)[2])
    assert pfx.prefix_pairs(L, b, bounds) < 0.6 * star_pairs


def test_pulsar_table_rejects_chunks_outside_their_block():
    with pytest.raises(ValueError):
        pfx.pulsar_table(256, 64, [np.array([2]), np.array([5]), np.array([0])], chunk=32, sink=8)


def test_pulsar_table_through_the_oracle_matches_dense_mask():
    L, b, chunk, sink = 96, 32, 4, 6
    chunks = pfx.draw_chunks(L, b, chunk=chunk, budget=0.25, sink=sink, seed=1)
    src, pos, bounds = pfx.pulsar_table(L, b, chunks, chunk=chunk, sink=sink)
    g = torch.Generator().manual_seed(4)
    q = torch.randn(1, L, 2, 8, generator=g).to(torch.bfloat16)
    k = torch.randn(1, L, 1, 8, generator=g).to(torch.bfloat16)
    v = torch.randn(1, L, 1, 8, generator=g).to(torch.bfloat16)
    hh, rr = np.meshgrid(np.arange(2), np.arange(L), indexing="ij")
    o, l, nvis = orc.phase1_gather_rows(q, k, v, b, src, pos, bounds, 1e4,
                                        np.zeros(hh.size), hh.ravel(), rr.ravel(), round_qk=False)
    lists = [[(int(s), int(s) + 1) for s in src[bounds[i][0]:bounds[i][1]]] for i in range(L // b)]
    M = brute.prefix_mask(L, b, lists)
    assert (nvis[:L] == M.sum(1)).all()
    qr_ = brute.rope_complex(q.double().numpy()[0], np.arange(L), 1e4)
    kr_ = brute.rope_complex(k.double().numpy()[0], np.arange(L), 1e4)
    ro, rl = brute.masked_attention(qr_[:, 0], kr_[:, 0], v.double().numpy()[0, :, 0], M)
    np.testing.assert_allclose(o[:L], ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l[:L], rl, rtol=0, atol=1e-12)
