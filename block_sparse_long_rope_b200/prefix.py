"""Prefix tables for star_phase1_encode_ext (host-side layout builders).

A prefix table has G rows; row g is context row src[g] (src >= 0) or given
row -1 - src[g], its key rotated at pos[g]; block i sees table rows
bounds[i, 0] .. bounds[i, 1] - 1, then itself causally.

- star_table: the Star anchor, the first a tokens at positions 0..a-1, seen
  by every block i >= 1 [pith 2WVXFXZ2, "What carries the argument"].
- shifted_anchor_table: the same rows at other position IDs (the anchor
  position ablation; atlas.scime.ai summary, measured-effects table).
- pulsar_table: a sink of the first tokens plus per-block summaries of
  fixed-size chunks, block i seeing [sink || Sigma_0 || ... || Sigma_{i-1}]
  with every row at its original global position [pith 2607.20457, "What
  carries the argument"]. Which chunks form a summary is the caller's choice
  (the pages score chunks by Max-IDF over token ids); draw_chunks gives a
  seeded draw of the same size for synthetic inputs.
"""
import numpy as np


def n_blocks(L, block_len):
    return -(-L // block_len)


def star_table(L, block_len, anchor_len):
    """(src, pos, bounds) of the Star anchor [0, anchor_len)."""
    n = n_blocks(L, block_len)
    src = np.arange(anchor_len, dtype=np.int32)
    bounds = np.zeros((n, 2), dtype=np.int32)
    bounds[1:] = (0, anchor_len)
    return src, src.copy(), bounds


def shifted_anchor_table(L, block_len, anchor_len, positions):
    """The Star anchor's rows at the given position IDs."""
    src, _, bounds = star_table(L, block_len, anchor_len)
    pos = np.asarray(positions, dtype=np.int64)
    if pos.shape != (anchor_len,):
        raise ValueError("one position per anchor row")
    return src, pos.astype(np.int32), bounds


def draw_chunks(L, block_len, chunk=32, budget=0.125, sink=64, seed=0):
    """Seeded stand-in for a chunk scorer: for every block but the last,
    round(budget * block_len / chunk) distinct chunk indices (of chunks that
    lie inside the block and outside the sink), ascending."""
    n = n_blocks(L, block_len)
    rng = np.random.default_rng(seed)
    per = max(1, int(round(budget * block_len / chunk)))
    out = []
    for j in range(n - 1):
        first = -(-sink // chunk) if j == 0 else 0
        cand = np.arange(first, block_len // chunk)
        out.append(np.sort(rng.choice(cand, size=min(per, cand.size), replace=False)))
    return out


def pulsar_table(L, block_len, chunks, chunk=32, sink=64):
    """(src, pos, bounds) of [sink || Sigma_0 || ... || Sigma_{i-1}]:
    chunks[j] lists the chunk indices (within block j, in positional order)
    that form Sigma_j; rows keep their original positions."""
    n = n_blocks(L, block_len)
    if len(chunks) < n - 1:
        raise ValueError("one chunk list per block before the last")
    rows = [np.arange(min(sink, L))]
    bounds = np.zeros((n, 2), dtype=np.int64)
    end = rows[0].size
    for i in range(1, n):
        j = i - 1
        for c in np.asarray(chunks[j], dtype=np.int64):
            s = j * block_len + c * chunk
            e = min(s + chunk, (j + 1) * block_len, L)
            if not (j * block_len <= s < e):
                raise ValueError(f"chunk {c} lies outside block {j}")
            rows.append(np.arange(s, e))
            end += e - s
        bounds[i] = (0, end)
    src = np.concatenate(rows).astype(np.int32)
    return src, src.copy(), bounds.astype(np.int32)


def prefix_pairs(L, block_len, bounds):
    """Visible (query, key) pairs of the generalised Phase 1: the causal
    pairs of every block plus rows-of-block-i x |slice i|."""
    n = n_blocks(L, block_len)
    total = 0
    for i in range(n):
        rows = min(block_len, L - i * block_len)
        total += rows * (rows + 1) // 2 + rows * max(0, int(bounds[i][1]) - int(bounds[i][0]))
    return total
