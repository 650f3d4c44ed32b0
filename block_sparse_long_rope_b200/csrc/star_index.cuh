// Index math of Star Attention, evaluated identically on host and device.
//
// Phase 1 [pith 2WVXFXZ2, "What carries the argument"; minor comment on
// Section 2.1]: context row r lies in block i = r / b. Block 0 (c'_1 = c_1)
// is plain causal over [0, r]. Block i >= 1 sees the anchor keys [0, a) at
// their original positions, then its own block causally: [i*b, r].
// Phase 2 [pith 2WVXFXZ2, Referee summary; abstract]: a new token at
// position p sees every context block in full (one split each) and the tail
// [L, p] causally.
//
// Work is cut into 128-row query tiles and 128-key KV tiles. Query tiles are
// aligned to their block start, so a tile never straddles two blocks.
#pragma once

#include <stdint.h>

namespace star {

constexpr int kTileM = 128;  // query rows per tile (tcgen05 M)
constexpr int kTileN = 128;  // keys per KV tile

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int imin(int a, int b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int imax(int a, int b) { return a > b ? a : b; }

// Visible key ranges of context row r in Phase 1: {anchor_lo, anchor_hi,
// own_lo, own_hi}, half-open; block 0 has an empty anchor range.
__host__ __device__ __forceinline__ void phase1_row_ranges(int r, int b, int a, int* out4) {
  int i = r / b;
  out4[0] = 0;
  out4[1] = (i == 0) ? 0 : a;
  out4[2] = i * b;
  out4[3] = r + 1;
}

// One contiguous run of KV tiles with a common visibility rule:
// key c is visible to a row at position p iff lo <= c < hi and, when causal,
// c <= p. Tiles start at key0 + kTileN * t, t in [0, ntiles).
struct KvSpan {
  int key0, ntiles, lo, hi, causal;
  int src;  // 0: the KV cache, 1: the gathered prefix table
};

// A unit of attention work: query rows [q_lo, q_hi) of one (batch, head
// slot group) and up to two KV spans, visited in order.
struct WorkItem {
  int b, kvh, slot0;      // batch, KV head, first query head of the group
  int q_lo, q_hi;         // query rows (rows of the rotated-Q buffer)
  int pos_base;           // position of query row q = pos_base + q
  int split;              // Phase-2 split written by this item (-1 in Phase 1)
  int nspan;
  KvSpan span[2];
  __host__ __device__ int ntiles() const {
    return span[0].ntiles + (nspan > 1 ? span[1].ntiles : 0);
  }
  __host__ __device__ void tile(int t, int* key0, int* lo, int* hi, int* causal) const {
    // field-wise selects keep the spans in registers
    const bool first = t < span[0].ntiles;
    const int tt = first ? t : t - span[0].ntiles;
    *key0 = (first ? span[0].key0 : span[1].key0) + tt * kTileN;
    *lo = first ? span[0].lo : span[1].lo;
    *hi = first ? span[0].hi : span[1].hi;
    *causal = first ? span[0].causal : span[1].causal;
  }
};

// Query chunks of at most 64 tokens fill a 128-row tile with two heads of
// the same GQA group (rows 0-63 one head, 64-127 the next), so no MMA row
// is left empty; needs four heads per KV head (two tiles of two heads).
__host__ __device__ __forceinline__ int chunk_heads_per_slot(int T, int Hq, int Hkv) {
  return (T <= 64 && (Hq / Hkv) % 4 == 0) ? 2 : 1;
}

// Geometry shared by the two attention modes. Query heads are handled
// `hpc` tiles at a time (the heads of one GQA group that share every K/V
// tile), each tile holding `hps` heads (2 only for short query chunks).
struct AttnGeom {
  int B, Hq, Hkv, hpc;  // hpc: query tiles (head slots) per CTA (1 or 2)
  int hps;              // heads per tile: 1, or 2 (64 rows each; Phase 2 only)
  int L, b, a;          // context length, block length, anchor length
  int n;                // context blocks = ceil(L / b)
  // Phase 2 only
  int T, tail_len;
  int tail;             // 1: the call's cache holds the tail split (new tokens)
  int nsub, sub_len;    // query chunks: sub-splits per context block, keys each

  __host__ __device__ int heads_per_item() const { return hpc * hps; }
  __host__ __device__ int groups() const { return B * Hkv * ((Hq / Hkv) / heads_per_item()); }
  __host__ __device__ int qtiles_full() const { return ceil_div(imin(b, L), kTileM); }
  __host__ __device__ int qtiles_last() const { return ceil_div(L - (n - 1) * b, kTileM); }

  // ---- Phase 1 -------------------------------------------------------------
  // Items are ordered by (batch, KV head) first, then block by block: the
  // anchor-carrying blocks 1..n-2, the last block, then block 0 (no anchor,
  // the shortest items). The CTAs in flight then read one KV head's anchor
  // and one block, 2 x 64 MB at 1M tokens, which L2 mostly keeps. Inside a
  // block the query tiles run longest first (descending index j, work grows
  // with j), the head groups of a tile next to each other.
  __host__ __device__ int phase1_pairs() const {  // (block, query tile) pairs
    int nf = qtiles_full(), nl = qtiles_last();
    return (nf - nl) * (n - 1) + nl * n;
  }
  __host__ __device__ int phase1_items() const { return phase1_pairs() * groups(); }
  __host__ __device__ void group_decode(int gi, WorkItem* w) const {
    int g = Hq / Hkv, per_kv = g / heads_per_item();
    w->b = gi / (Hkv * per_kv);
    int rem = gi % (Hkv * per_kv);
    w->kvh = rem / per_kv;
    w->slot0 = w->kvh * g + (rem % per_kv) * heads_per_item();
  }
  __host__ __device__ WorkItem phase1_item(int item) const {
    const int per_kv = (Hq / Hkv) / heads_per_item();  // head groups of one KV head
    const int chunk = phase1_pairs() * per_kv;
    const int bk = item / chunk;          // b * Hkv + kvh
    const int in = item % chunk;
    const int nf = qtiles_full(), nl = qtiles_last();
    int i, j, r;
    if (n == 1) {
      i = 0;
      r = in;
      j = nl - 1 - r / per_kv;
    } else {
      const int full = (n - 2) * nf * per_kv, last = nl * per_kv;
      if (in < full) {  // blocks 1..n-2
        i = 1 + in / (nf * per_kv);
        r = in % (nf * per_kv);
        j = nf - 1 - r / per_kv;
      } else if (in < full + last) {  // block n-1
        i = n - 1;
        r = in - full;
        j = nl - 1 - r / per_kv;
      } else {  // block 0
        i = 0;
        r = in - full - last;
        j = nf - 1 - r / per_kv;
      }
    }
    const int sg = r % per_kv;
    const int gi = bk * per_kv + sg;
    WorkItem w;
    group_decode(gi, &w);
    int s = i * b, e = imin(s + b, L);
    w.q_lo = s + j * kTileM;
    w.q_hi = imin(w.q_lo + kTileM, e);
    w.pos_base = 0;
    w.split = -1;
    // own block: tiles aligned to the block start, up to the diagonal tile
    const KvSpan own{s, j + 1, s, L, 1, 0};
    if (i > 0 && a > 0) {
      w.span[0] = KvSpan{0, ceil_div(a, kTileN), 0, a, 0, 0};  // the anchor c_1
      w.span[1] = own;
      w.nspan = 2;
    } else {
      w.span[0] = own;
      w.span[1] = KvSpan{0, 0, 0, 0, 0, 0};
      w.nspan = 1;
    }
    return w;
  }

  // ---- Phase 2 (query chunk, partial mode) ---------------------------------
  // Items: split-major (context blocks 0..n-1, each cut into nsub equal
  // sub-splits of sub_len keys, then the tail), then query tile, then head
  // group. Item split index s < n*nsub is sub-split s % nsub of block s / nsub.
  __host__ __device__ int phase2_qtiles() const { return ceil_div(T, kTileM); }
  __host__ __device__ int phase2_splits() const { return n * nsub + tail; }
  __host__ __device__ int phase2_items() const { return phase2_splits() * phase2_qtiles() * groups(); }
  __host__ __device__ WorkItem phase2_item(int item) const {
    int G = groups(), nq = phase2_qtiles();
    int split = item / (nq * G);
    int rem = item % (nq * G);
    int j = rem / G;
    WorkItem w;
    group_decode(rem % G, &w);
    w.q_lo = j * kTileM;
    w.q_hi = imin(w.q_lo + kTileM, T);
    w.pos_base = L + tail_len;
    w.split = split;
    w.nspan = 1;
    w.span[1] = KvSpan{0, 0, 0, 0, 0, 0};
    if (split < n * nsub) {
      const int blk = split / nsub, sub = split % nsub;
      int s = blk * b + sub * sub_len, e = imin(imin(s + sub_len, (blk + 1) * b), L);
      w.span[0] = KvSpan{s, ceil_div(e - s, kTileN), s, e, 0, 0};
    } else {
      // tail keys [L, L + tail_len + T); this tile's last row sits at
      // position L + tail_len + q_hi - 1
      int last = tail_len + w.q_hi;  // keys needed: [L, L + last)
      w.span[0] = KvSpan{L, ceil_div(last, kTileN), L, L + tail_len + T, 1, 0};
    }
    return w;
  }
};

}  // namespace star
