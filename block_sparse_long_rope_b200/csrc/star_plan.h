// Host-side work planning of the Phase-2 kernels, shared by the C ABI and
// its CPU tests: decode work units (keys per CTA unit, units per split) and
// the query-chunk sub-split rule. Host code only.
#pragma once

#include <algorithm>

#include "star_kernels.cuh"

namespace star {

// Decode path scratch: per (batch, KV head), chunk partials of kDecRows rows.
inline int decode_chunks_per_head(int L, int b, int n, int tail_plus_T, int chunk, int* nc_full,
                                  int* nc_last, int* nc_tail) {
  *nc_full = ceil_div(imin(b, L), chunk);
  *nc_last = ceil_div(L - (n - 1) * b, chunk);
  *nc_tail = ceil_div(tail_plus_T, chunk);
  return (n - 1) * *nc_full + *nc_last + *nc_tail;
}

// Keys per decode work unit (a multiple of the 64-key tile). The grid is two
// persistent CTAs per SM; units are sized so that all of them fit in that
// one wave with equal work (the total tiles of all splits divided over the
// CTAs left after one extra unit per split for the ragged ends), and so that
// a split has at most kMaxChunksPerSplit units. When there are more splits
// than CTAs every split is one unit and CTAs loop over several.
inline int decode_chunk(int B, int Hkv, int L, int b, int n, int nsplit, int tail_plus_T, int sms) {
  const int tile = kDecTile;
  const long long tiles_head = (long long)(n - 1) * ceil_div(imin(b, L), tile) +
                               ceil_div(L - (n - 1) * b, tile) + ceil_div(tail_plus_T, tile);
  const long long total_tiles = tiles_head * B * Hkv;
  const long long splits = (long long)B * Hkv * nsplit;
  const long long ctas = 2ll * sms;
  const long long room = ctas - splits;
  const int max_split_tiles = ceil_div(imax(imin(b, L), tail_plus_T), tile);
  long long chunk_tiles = room > 0 ? (total_tiles + room - 1) / room : max_split_tiles;
  chunk_tiles = std::max<long long>(chunk_tiles, ceil_div(max_split_tiles, kMaxChunksPerSplit));
  chunk_tiles = std::max<long long>(1, std::min<long long>(chunk_tiles, max_split_tiles));
  // equal units within a full block: the same number of units, none ragged
  // (64 tiles in chunks of 9 would leave a 1-tile unit; 8 x 8 balances them).
  // Kept only if the split limit holds and the unit count stays within one
  // wave (or the count before), which the scratch size assumes.
  const long long block_tiles = ceil_div(imin(b, L), tile);
  const long long last_tiles = ceil_div(L - (n - 1) * b, tile);
  const long long tail_tiles = ceil_div(tail_plus_T, tile);
  auto units_for = [&](long long ct) {
    return (long long)B * Hkv *
           ((n - 1) * ((block_tiles + ct - 1) / ct) + (last_tiles + ct - 1) / ct +
            (tail_tiles + ct - 1) / ct);
  };
  const long long per_block = (block_tiles + chunk_tiles - 1) / chunk_tiles;
  const long long even = std::max<long long>(
      (block_tiles + per_block - 1) / per_block,
      ceil_div(max_split_tiles, kMaxChunksPerSplit));
  if (units_for(even) <= std::max(units_for(chunk_tiles), ctas)) chunk_tiles = even;
  return static_cast<int>(chunk_tiles) * tile;
}

inline bool use_decode_path(int T, int Hq, int Hkv) {
  const int g = Hq / Hkv;
  return T * g <= kDecRows;
}

// Units decode_chunk can make for any context with L + tail <= Lcap: at
// most max(2 * SMs, splits) + splits (one extra per split for its ragged
// end), with at most 256 SMs. The decode scratch is sized for this many.
inline long long decode_units_bound(int B, int Hkv, int Lcap, int block_len) {
  const long long splits = (long long)B * Hkv * (ceil_div(Lcap, block_len) + 1);
  return std::max<long long>(512, splits) + splits;
}

// Query chunks (tensor-core path): sub-splits per context block. A call with
// fewer (split, query tile, head group) items than one wave of a B200 (148
// CTAs) cuts every block into nsub equal sub-splits (a multiple of 128 keys,
// at most 4), so more SMs share the work; the sub-split partials are then
// reduced into the per-split partials. Only whole blocks (L a multiple of
// block_len) and calls with the tail split are cut. Depends on the shape
// only, so the workspace size can be computed without a device.
inline int chunk_subsplits(int B, int Hq, int Hkv, int T, int L, int block_len, int with_tail) {
  constexpr long long kWave = 148;
  if (!with_tail || L % block_len != 0) return 1;
  const int n = L / block_len;
  const int g = Hq / Hkv, hpc = (g % 2 == 0) ? 2 : 1;
  const int hpi = hpc * chunk_heads_per_slot(T, Hq, Hkv);
  const long long per_split = (long long)B * Hkv * (g / hpi) * ceil_div(T, 128);
  if ((n + 1) * per_split >= kWave) return 1;
  int nsub = (int)std::min<long long>(4, (kWave - per_split) / (n * per_split));
  while (nsub > 1 && block_len % (nsub * 128) != 0) --nsub;
  return std::max(1, nsub);
}

}  // namespace star
