"""The attention kernels' work decomposition (star_index.cuh, built here for
the host) against the visibility rule of Star Attention, on CPU.

Phase 1 [pith 2WVXFXZ2, "What carries the argument"; minor comment on
Section 2.1]: context row r of block i = r // b sees keys [0, r] when i = 0,
else the anchor [0, a) and its own block [i*b, r]. Phase 2 [pith 2WVXFXZ2,
Referee summary; abstract]: a new token sees every context block in full,
one split each (or each of its sub-splits), and the tail [L, p] causally.

Every (batch, query head, row) must belong to exactly one work item, and the
keys an item's spans make visible to a row (its 128-key tiles, filtered by
each span's [lo, hi) and causal rule) must be exactly the keys the rule
gives: a missing key changes the softmax, an extra one attends outside the
block."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_long_rope_b200", "csrc")
TILE = 128


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("wi") / "libwi.so")
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-shared", "-fPIC", "-I" + CSRC,
                           os.path.join(ROOT, "tests", "harness", "work_items.cpp"), "-o", out])
    lb = ctypes.CDLL(out)
    for f in ("wi_phase1_item", "wi_phase2_item"):
        getattr(lb, f).restype = None
    return lb


def _item(fn, *args):
    buf = (ctypes.c_int * 20)()
    fn(*[ctypes.c_int(int(v)) for v in args], buf)
    v = list(buf)
    spans = [dict(key0=v[8 + 6 * s], ntiles=v[9 + 6 * s], lo=v[10 + 6 * s], hi=v[11 + 6 * s],
                  causal=v[12 + 6 * s], src=v[13 + 6 * s]) for s in range(v[7])]
    return dict(b=v[0], kvh=v[1], slot0=v[2], q_lo=v[3], q_hi=v[4], pos_base=v[5], split=v[6],
                spans=spans)


def _span_visibility(it, rows, nkeys):
    """[len(rows), nkeys] bool: the keys each row sees through the item's spans."""
    vis = np.zeros((len(rows), nkeys), dtype=bool)
    pos = it["pos_base"] + rows
    for sp in it["spans"]:
        keys = sp["key0"] + np.arange(sp["ntiles"] * TILE)
        keys = keys[(keys >= sp["lo"]) & (keys < sp["hi"])]
        assert keys.size == 0 or (keys.min() >= 0 and keys.max() < nkeys)
        ok = np.ones((len(rows), keys.size), dtype=bool)
        if sp["causal"]:
            ok &= keys[None, :] <= pos[:, None]
        # a key seen through two spans would be counted twice in the softmax
        assert not (vis[:, keys] & ok).any()
        vis[:, keys] |= ok
    return vis


PHASE1 = [  # (B, Hq, Hkv, L, b, a)
    (1, 4, 1, 2048, 512, 512),
    (2, 4, 2, 1000, 300, 100),
    (1, 3, 3, 777, 256, 200),
    (1, 2, 1, 640, 128, 0),
    (1, 2, 2, 500, 1024, 0),
    (1, 8, 2, 1536, 512, 128),
    (1, 4, 2, 500, 64, 64),
    (1, 2, 1, 100, 1, 1),
    (1, 16, 2, 1300, 650, 650),
    (2, 16, 4, 1100, 256, 256),   # items ordered KV-head-major over two sequences
]


@pytest.mark.parametrize("geo", PHASE1, ids=[f"L{g[3]}b{g[4]}a{g[5]}g{g[1] // g[2]}" for g in PHASE1])
def test_phase1_items_cover_each_row_once_with_exactly_its_visible_keys(lib, geo):
    B, Hq, Hkv, L, b, a = geo
    hpc = lib.wi_hpc(Hq, Hkv)
    n_items = lib.wi_phase1_items(B, Hq, Hkv, L, b, a)
    count = np.zeros((B, Hq, L), dtype=np.int64)
    rows_all = np.arange(L)
    blk = rows_all // b
    for i in range(n_items):
        it = _item(lib.wi_phase1_item, B, Hq, Hkv, L, b, a, i)
        assert it["split"] == -1 and it["pos_base"] == 0
        assert it["q_hi"] - it["q_lo"] <= TILE and it["q_lo"] < it["q_hi"] <= L
        # a query tile never straddles two blocks
        assert it["q_lo"] // b == (it["q_hi"] - 1) // b
        heads = range(it["slot0"], it["slot0"] + hpc)
        assert all(h // (Hq // Hkv) == it["kvh"] for h in heads)
        rows = np.arange(it["q_lo"], it["q_hi"])
        for h in heads:
            count[it["b"], h, rows] += 1
        want = np.zeros((len(rows), L), dtype=bool)
        keys = np.arange(L)
        for k, r in enumerate(rows):
            i_blk = blk[r]
            if i_blk == 0:
                want[k] = keys <= r
            else:
                want[k] = (keys < a) | ((keys >= i_blk * b) & (keys <= r))
        got = _span_visibility(it, rows, L)
        assert np.array_equal(got, want), (i, it)
    assert (count == 1).all()


@pytest.mark.parametrize("geo", [(2, 16, 4, 1100, 256, 256), (1, 32, 8, 1 << 20, 131072, 131072),
                                 (1, 8, 2, 1536, 512, 128)],
                         ids=["B2-ragged", "llama8b-1m", "a<b"])
def test_phase1_item_order_keeps_one_kv_head_and_block_together(lib, geo):
    """The L2-friendly order: items run (batch, KV head) by (batch, KV head);
    inside one, block by block (1..n-2, the last block, then block 0); inside
    a block, query tiles longest first."""
    B, Hq, Hkv, L, b, a = geo
    n = -(-L // b)
    n_items = lib.wi_phase1_items(B, Hq, Hkv, L, b, a)
    want_blocks = list(range(1, n - 1)) + ([n - 1] if n > 1 else []) + [0]
    step = max(1, n_items // 20000)  # the 1M shape has 131072 items: a sample and its neighbours
    idx = range(0, n_items) if n_items <= 20000 else sorted(
        set(range(0, n_items, step)) | set(range(1, n_items, step)))
    order = []
    for i in idx:
        it = _item(lib.wi_phase1_item, B, Hq, Hkv, L, b, a, i)
        order.append((i, it["b"] * Hkv + it["kvh"], it["q_lo"] // b, it["q_lo"]))
    # (batch, KV head) never decreases
    assert all(x[1] <= y[1] for x, y in zip(order, order[1:]))
    for bk in sorted({o[1] for o in order}):
        seq = [o for o in order if o[1] == bk]
        blk_seq = [o[2] for o in seq]
        # blocks appear as contiguous runs, in the stated order
        runs = [blk_seq[0]] + [y for x, y in zip(blk_seq, blk_seq[1:]) if y != x]
        assert runs == [blk for blk in want_blocks if blk in set(blk_seq)], runs[:12]
        # inside a block, query tiles never move forward
        for x, y in zip(seq, seq[1:]):
            if x[2] == y[2] and y[0] == x[0] + 1:
                assert y[3] <= x[3]


PHASE2 = [  # (B, Hq, Hkv, L, b, T, tail_len, with_tail, nsub)
    (1, 4, 1, 2048, 512, 16, 0, 1, 1),
    (2, 4, 2, 1000, 300, 20, 5, 1, 1),
    (1, 16, 2, 700, 256, 3, 7, 1, 1),
    (1, 2, 2, 900, 200, 130, 1, 1, 1),
    (1, 32, 8, 4096, 1024, 128, 0, 1, 2),
    (1, 32, 8, 16384, 4096, 128, 0, 1, 4),
    (1, 4, 2, 1024, 256, 40, 3, 0, 1),   # a shard without the tail split
    (2, 32, 8, 2048, 512, 64, 9, 1, 2),  # 64 tokens: two heads per tile, sub-splits
    (1, 8, 1, 1100, 256, 33, 0, 1, 1),   # ragged last block, two heads per tile
]


@pytest.mark.parametrize("geo", PHASE2, ids=[f"L{g[3]}b{g[4]}T{g[5]}sub{g[8]}tail{g[7]}" for g in PHASE2])
def test_phase2_items_cover_each_split_row_once_with_exactly_its_keys(lib, geo):
    B, Hq, Hkv, L, b, T, tail_len, with_tail, nsub = geo
    hpi = lib.wi_phase2_heads_per_item(Hq, Hkv, T)  # 4 for <= 64 tokens and groups of 4+
    assert hpi == lib.wi_hpc(Hq, Hkv) * (2 if T <= 64 and (Hq // Hkv) % 4 == 0 else 1)
    n = -(-L // b)
    sub_len = b // nsub
    n_items = lib.wi_phase2_items(*geo)
    nsplit = lib.wi_phase2_splits(*geo)
    assert nsplit == n * nsub + with_tail
    count = np.zeros((B, Hq, nsplit, T), dtype=np.int64)
    nkeys = L + tail_len + T
    for i in range(n_items):
        it = _item(lib.wi_phase2_item, *geo, i)
        s = it["split"]
        assert 0 <= s < nsplit and it["pos_base"] == L + tail_len
        assert it["q_lo"] < it["q_hi"] <= T and it["q_hi"] - it["q_lo"] <= TILE
        rows = np.arange(it["q_lo"], it["q_hi"])
        assert it["slot0"] % hpi == 0 and it["kvh"] == it["slot0"] // (Hq // Hkv)
        for h in range(it["slot0"], it["slot0"] + hpi):
            count[it["b"], h, s, rows] += 1
        keys = np.arange(nkeys)
        if s < n * nsub:
            lo = (s // nsub) * b + (s % nsub) * sub_len
            hi = min(lo + sub_len, (s // nsub + 1) * b, L)
            want = np.broadcast_to((keys >= lo) & (keys < hi), (len(rows), nkeys))
        else:
            pos = L + tail_len + rows
            want = (keys[None, :] >= L) & (keys[None, :] <= pos[:, None])
        got = _span_visibility(it, rows, nkeys)
        assert np.array_equal(got, want), (i, it)
    assert (count == 1).all()
    # the sub-splits of a block partition it: together they are one split per block
    if nsub > 1:
        for blk in range(n):
            parts = [(blk * b + u * sub_len, min(blk * b + (u + 1) * sub_len, (blk + 1) * b, L))
                     for u in range(nsub)]
            assert parts[0][0] == blk * b and parts[-1][1] == min((blk + 1) * b, L)
            assert all(p[1] == q[0] for p, q in zip(parts, parts[1:]))


def test_rope_unit_index_by_multiply_high_is_exact_for_every_head_count():
    """The RoPE kernel splits a unit u = t * per_tok + rem (token, then head and
    16-byte chunk) with one multiply-high by magic = floor((2^32 - 1) / per_tok)
    + 1 instead of a division; per_tok = H * D / 16 for H <= 2048 heads and a
    CTA covers 8 tokens, so u < 8 * per_tok. Checked here against integer
    division for every head count and both head sizes, every u."""
    for D in (64, 128):
        cpr = D // 16
        for H in range(1, 2049):
            d = H * cpr
            magic = (0xFFFFFFFF // d) + 1
            u = np.arange(8 * d, dtype=np.uint64)
            t = (u * np.uint64(magic)) >> np.uint64(32)
            assert np.array_equal(t, u // np.uint64(d)), (D, H)
