// Block-sparse causal flash attention on 5th-generation tensor cores
// (tcgen05 + tensor memory + TMA), sm_100a.
//
// Phase 1 of Star Attention: context block i >= 1 attends to the anchor
// block c_1 (original positions) and causally to itself; block 0 is plain
// causal [pith 2WVXFXZ2, "What carries the argument"; minor comment on
// Section 2.1]. On one GPU the pages' hosts become work items processed in
// parallel. The anchor's K/V are exactly the cache rows of block 0 (same
// tokens, same positions, one layer), so every block reads those shared rows
// instead of recomputing and storing an anchor copy.
//
// The same kernel in "partial" mode computes Phase-2 query chunks: each item
// attends to one split (a context block in full, or the causal tail) and
// writes a split-normalised fp32 output plus its LSE [pith 2WVXFXZ2, Referee
// summary].
//
// Work item = (batch, GQA group slice of `hpc` query heads, query tile of
// 128 rows). Only the KV tiles a tile can see are visited: the anchor tiles
// (no mask unless ragged) and the own-block tiles up to the diagonal (causal
// mask on the diagonal only); everything else is skipped. The hpc (<= 2)
// heads of one KV head share each K/V tile in shared memory (GQA reuse).
//
// Warp roles (320 threads, one CTA per SM):
//   warps 0-3  softmax of head slot 0 (thread = query row = TMEM lane)
//   warps 4-7  softmax of head slot 1
//   warp 8     TMA producer (Q once, then K and V tiles through a ring)
//   warp 9     TMEM allocator and single-thread tcgen05.mma issuer
// Tensor memory (512 columns): S0 | S1 | O0 | O1. P (bf16) overwrites the
// first 64 columns of its S and feeds the P*V MMA straight from TMEM.
// MMA order per KV tile t: PV0(t), S0(t+1), PV1(t), S1(t+1), so slot 0's
// softmax of tile t+1 overlaps slot 1's MMAs and vice versa.
// Online softmax in the exp2 domain with the 1/sqrt(D) scale folded in; the
// running max is only moved (and O rescaled in TMEM) when it grows by more
// than 2^8, which keeps every P <= 256 and the result exact.
#include <math.h>

#include "star_common.cuh"
#include "star_kernels.cuh"

namespace star {

namespace {

template <int D>
struct AttnCfg {
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kHalf = 128 * 128;          // one 64-column TMA box of a 128-row tile
  static constexpr int kTile = kHalf * (D / 64);   // a Q, K or V tile
  static constexpr int kOffQ = 0;                  // two Q tiles
  static constexpr int kOffK = 2 * kTile;
  static constexpr int kOffV = kOffK + kStages * kTile;
  static constexpr int kOffBar = kOffV + kStages * kTile;
  static constexpr int kBytes = kOffBar + 256 + 1024;  // + barriers + alignment slack
  // tensor-memory columns of S and O for head slot x
  __device__ static constexpr uint32_t col_s(int x) { return 128u * static_cast<uint32_t>(x); }
  __device__ static constexpr uint32_t col_o(int x) { return 256u + D * static_cast<uint32_t>(x); }
  static constexpr uint32_t kTmemCols = 512;
};

constexpr int kAttnThreads = 320;

// ---- Phase-2 query chunks: where an item's rows go ---------------------------
// An item of a block cut into sub-splits (nsub > 1) writes sub-split row
// (b, head, split, qrow) of sub_o / sub_lse (chunk_finish_kernel reduces
// them); any other item (a whole block, or the tail) writes its split's row
// of part_o / part_lse directly. Returns the row index; *to_sub tells which
// pair of buffers it indexes.
__device__ __forceinline__ size_t p2_row(const AttnParams& p, const WorkItem& w, int head, int qrow,
                                         bool* to_sub) {
  const AttnGeom& g = p.geom;
  const size_t bh = static_cast<size_t>(w.b) * g.Hq + head;
  *to_sub = g.nsub > 1 && w.split < g.n * g.nsub;
  if (*to_sub) return (bh * (g.n * g.nsub) + w.split) * g.T + qrow;
  const int api = (w.split < g.n * g.nsub) ? w.split / g.nsub : g.n;
  return (bh * p.nsplit + api) * g.T + qrow;
}

constexpr uint64_t kDrainNs = 100000000ull;  // 100 ms

__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > limit_ns) return;
  }
}

}  // namespace

// kMode 0: Phase 1; kMode 1: Phase-2 query chunk (one instantiation each,
// so Phase 1 carries none of the query chunk's epilogue code).
template <int D, int kMode>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_kernel(const __grid_constant__ AttnParams p) {
  using C = AttnCfg<D>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* q_full = reinterpret_cast<uint64_t*>(sm + C::kOffBar);
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + S;
  uint64_t* v_full = k_empty + S;
  uint64_t* v_empty = v_full + S;
  uint64_t* s_full = v_empty + S;  // [2]
  uint64_t* p_full = s_full + 2;   // [2]
  uint64_t* o_full = p_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_full + 1);
  __shared__ volatile int abort_flag;
  __shared__ KvSpan s_span[2];  // the KV spans this item visits, in order
  __shared__ int s_nspan, s_nkv;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WorkItem w = (kMode == 0) ? p.geom.phase1_item(blockIdx.x) : p.geom.phase2_item(blockIdx.x);
  const int hpc = p.geom.hpc;
  // heads per 128-row tile: 2 for query chunks of at most 64 tokens (rows
  // 0-63 head slot0 + 2x, rows 64-127 the next head), else 1
  const int hps = (kMode == 1) ? p.geom.hps : 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 128);
    }
    mbar_init(o_full, 1);
    fence_barrier_init();
    abort_flag = 0;
    // span list: the item's own spans, or in ext mode the block's slice of
    // the prefix table (clamped to the table; a slice outside it is recorded
    // as a bounds error) and the own block
    int ns = 0;
    if (kMode == 0 && p.ext) {
      const int blk = w.q_lo / p.geom.b;
      if (p.bounds) {
        int gs = p.bounds[2 * blk], ge = p.bounds[2 * blk + 1];
        if (gs < 0 || ge > p.G || ge < gs) {
          atomicOr(p.status, kDevBounds);
          gs = imin(imax(gs, 0), p.G);
          ge = imin(imax(ge, gs), p.G);
        }
        if (ge > gs) s_span[ns++] = KvSpan{gs, ceil_div(ge - gs, kTileN), gs, ge, 0, 1};
      }
      s_span[ns++] = w.span[w.nspan - 1];  // own block, causal
    } else {
      for (int t = 0; t < w.nspan; ++t)
        if (w.span[t].ntiles > 0) s_span[ns++] = w.span[t];
    }
    int nt = 0;
    for (int t = 0; t < ns; ++t) nt += s_span[t].ntiles;
    s_nspan = ns;
    s_nkv = nt;
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nkv = s_nkv;

  if (warp == 8) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&p.tmQ);
      prefetch_tmap(&p.tmK);
      prefetch_tmap(&p.tmV);
      if (p.ext && p.G > 0) {
        prefetch_tmap(&p.tmKP);
        prefetch_tmap(&p.tmVP);
      }
      mbar_arrive_expect_tx(q_full, hpc * C::kTile);
      for (int x = 0; x < hpc; ++x)
        for (int hh = 0; hh < hps; ++hh)  // a 64-row box per head when hps = 2
#pragma unroll
          for (int hd = 0; hd < D / 64; ++hd)
            tma_load_4d(sm + C::kOffQ + x * C::kTile + hd * C::kHalf + hh * (C::kHalf / 2), &p.tmQ,
                        q_full, hd * 64, w.slot0 + x * hps + hh, w.q_lo, w.b);
      const int bz = w.b * p.geom.Hkv + w.kvh;
      int issued_k = 0, issued_v = 0;
      int csi = 0, cti = 0;  // span cursor
      for (int it = 0; it < nkv; ++it) {
        const int st = it % S, use = it / S;
        const KvSpan& sp = s_span[csi];
        const int key0 = sp.key0 + cti * kTileN;
        const CUtensorMap* mk = sp.src ? &p.tmKP : &p.tmK;
        const CUtensorMap* mv = sp.src ? &p.tmVP : &p.tmV;
        if (++cti == sp.ntiles) {
          ++csi;
          cti = 0;
        }
        if (use > 0 && !mbar_wait(&k_empty[st], (use - 1) & 1, &abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&k_full[st], C::kTile);
#pragma unroll
        for (int hd = 0; hd < D / 64; ++hd)
          tma_load_3d(sm + C::kOffK + st * C::kTile + hd * C::kHalf, mk, &k_full[st], hd * 64,
                      key0, bz);
        ++issued_k;
        if (use > 0 && !mbar_wait(&v_empty[st], (use - 1) & 1, &abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&v_full[st], C::kTile);
#pragma unroll
        for (int hd = 0; hd < D / 64; ++hd)
          tma_load_3d(sm + C::kOffV + st * C::kTile + hd * C::kHalf, mv, &v_full[st], hd * 64,
                      key0, bz);
        ++issued_v;
      }
      if (abort_flag) {  // let copies still in flight land before the CTA exits
        mbar_drain(q_full, 0, kDrainNs);
        for (int it = imax(0, issued_k - S); it < issued_k; ++it)
          mbar_drain(&k_full[it % S], (it / S) & 1, kDrainNs);
        for (int it = imax(0, issued_v - S); it < issued_v; ++it)
          mbar_drain(&v_full[it % S], (it / S) & 1, kDrainNs);
      }
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(128, 128, 0, 0);  // S = Q K^T, both K-major
      const uint32_t idO = idesc_bf16(128, D, 0, 1);    // O += P V, V is N-major
      const uint32_t q_base = smem_u32(sm + C::kOffQ);
      const uint32_t k_base = smem_u32(sm + C::kOffK);
      const uint32_t v_base = smem_u32(sm + C::kOffV);
      auto qk_desc = [&](uint32_t tile_base, int kk) {
        // K-major, 128-byte rows; 16-element k-steps move 32 bytes inside a
        // swizzle atom, every 4 k-steps move to the next 64-column box
        return sdesc_sw128(tile_base + (kk >> 2) * C::kHalf + (kk & 3) * 32, 16, 1024);
      };
      auto issue_s = [&](int x, int st) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + C::col_s(x), qk_desc(q_base + x * C::kTile, kk),
                 qk_desc(k_base + st * C::kTile, kk), idS, kk > 0 ? 1u : 0u);
        mma_commit(&s_full[x]);
      };
      bool ok = mbar_wait(q_full, 0, &abort_flag, p.status);
      if (ok) ok = mbar_wait(&k_full[0], 0, &abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        for (int x = 0; x < hpc; ++x) issue_s(x, 0);
        mma_commit(&k_empty[0]);
      }
      for (int it = 0; ok && it < nkv; ++it) {
        const int st = it % S, ph = (it / S) & 1;
        const bool has_next = it + 1 < nkv;
        const int nst = (it + 1) % S, nph = ((it + 1) / S) & 1;
        if (has_next && !mbar_wait(&k_full[nst], nph, &abort_flag, p.status)) break;
        if (!mbar_wait(&v_full[st], ph, &abort_flag, p.status)) break;
        tc_fence_after();
        for (int x = 0; x < hpc && ok; ++x) {
          if (!mbar_wait(&p_full[x], it & 1, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t vt = v_base + st * C::kTile;
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk)
            mma_ts(tmem + C::col_o(x), tmem + C::col_s(x) + kk * 8,
                   sdesc_sw128(vt + kk * 2048, C::kHalf, 1024), idO, (it > 0 || kk > 0) ? 1u : 0u);
          if (has_next) issue_s(x, nst);
        }
        if (!ok) break;
        if (has_next) mma_commit(&k_empty[nst]);
        mma_commit(&v_empty[st]);
      }
      // O complete (or abandoned): the final commit also drains every MMA in
      // flight before tensor memory is released
      mma_commit(o_full);
      mbar_drain(o_full, 0, kDrainNs);
    }
    __syncwarp();
  } else if ((warp >> 2) < hpc) {
    // ---------------------------------------------------------------- softmax
    const int x = warp >> 2;
    const int qw = warp & 3;
    const int row = qw * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(qw * 32) << 16;
    const uint32_t tS = tmem + lane_bits + C::col_s(x);
    const uint32_t tO = tmem + lane_bits + C::col_o(x);
    const int hrow = (hps == 2) ? (row >> 6) : 0;  // which head of the tile
    const int qrow = w.q_lo + ((hps == 2) ? (row & 63) : row);
    const int qpos = w.pos_base + qrow;
    const int min_pos = w.pos_base + w.q_lo;
    const float c = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;

    int csi = 0, cti = 0;  // span cursor
    for (int it = 0; it < nkv; ++it) {
      if (!mbar_wait(&s_full[x], it & 1, &abort_flag, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld32(tS + 32 * q, sr[q]);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q) reg_fence32(sr[q]);

      const KvSpan& sp = s_span[csi];
      const int key0 = sp.key0 + cti * kTileN, lo = sp.lo, hi = sp.hi, causal = sp.causal;
      if (++cti == sp.ntiles) {
        ++csi;
        cti = 0;
      }
      const bool full_vis =
          key0 >= lo && key0 + 128 <= hi && (!causal || key0 + 127 <= min_pos);
      if (!full_vis) {
        // the row's visible keys in this tile are one run [vlo, vhi) of
        // tile columns: one unsigned compare per column
        const int vlo = imax(lo - key0, 0);
        const int vhi = imin(imin(hi - key0, 128), causal ? qpos - key0 + 1 : 128);
        const uint32_t span = static_cast<uint32_t>(imax(vhi - vlo, 0));
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (static_cast<uint32_t>(32 * q + j - vlo) >= span) sr[q][j] = __float_as_uint(-INFINITY);
      }
      // row max: eight independent chains of 3-input max, then a tree (one
      // chain of 128 dependent max operations would dominate the latency)
      float mx[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) mx[j] = -INFINITY;
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < 16; ++j)
          mx[j & 7] = fmax3(mx[j & 7], __uint_as_float(sr[q][2 * j]), __uint_as_float(sr[q][2 * j + 1]));
      const float mt = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmaxf(fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const float m_new = fmaxf(m_run, mt);
      if (it == 0) {
        m_run = m_new;
      } else {
        const bool need = (m_new - m_run) * c > 8.f;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2_approx((m_run - m_new) * c) : 1.f;
#pragma unroll 1
          for (int q = 0; q < D / 16; ++q) {
            uint32_t r[16];
            tmem_ld16(tO + 16 * q, r);
            tmem_wait_ld();
            reg_fence16(r);
#pragma unroll
            for (int j = 0; j < 16; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
            tmem_st16(tO + 16 * q, r);
          }
          tmem_wait_st();
          l_run *= alpha;
          if (need) m_run = m_new;
        }
      }
      const float ref = (m_run == -INFINITY) ? 0.f : m_run * c;
      // x = s * c - ref for two keys at once (fma.rn.f32x2), exp2 on the MUFU
      // unit, row sums in four packed accumulators. P (bf16 pairs) goes back
      // over the first 64 columns of S, 32 keys at a time; S columns 16q..
      // are already consumed when quarter q is written.
      const uint64_t cc = f2_pack(c, c), nref = f2_pack(-ref, -ref);
      uint64_t ls[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[q][2 * j]), __uint_as_float(sr[q][2 * j + 1])),
                           cc, nref), x0, x1);
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          ls[j & 3] = f2_add(ls[j & 3], f2_pack(p0, p1));
          pk[j] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + 16 * q, pk);
      }
      float lsum = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float a, b;
        f2_unpack(ls[k], a, b);
        lsum += a + b;
      }
      l_run += lsum;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[x]);
    }

    // ---------------------------------------------------------------- epilogue
    if (ok && mbar_wait(o_full, 0, &abort_flag, p.status)) {
      tc_fence_after();
      const int head = w.slot0 + x * hps + hrow;
      const bool valid = qrow < w.q_hi;
      const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
      const int b = w.b;
      const int Hq = p.geom.Hq;
      for (int q = 0; q < D / 32; ++q) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld32(tO + 32 * q, r);
        tmem_wait_ld();
        reg_fence32(r);
        if (valid && kMode == 0) {
          __nv_bfloat16* dst =
              p.o + ((static_cast<size_t>(b) * p.geom.L + qrow) * Hq + head) * D + 32 * q;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 pkd;
            pkd.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]) * inv, __uint_as_float(r[8 * v + 1]) * inv);
            pkd.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]) * inv, __uint_as_float(r[8 * v + 3]) * inv);
            pkd.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]) * inv, __uint_as_float(r[8 * v + 5]) * inv);
            pkd.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]) * inv, __uint_as_float(r[8 * v + 7]) * inv);
            reinterpret_cast<uint4*>(dst)[v] = pkd;
          }
        } else if (valid) {
          bool to_sub;
          const size_t orow = p2_row(p, w, head, qrow, &to_sub);
          float* dst = (to_sub ? p.sub_o : p.part_o) + orow * D + 32 * q;
#pragma unroll
          for (int v = 0; v < 8; ++v)
            reinterpret_cast<float4*>(dst)[v] =
                make_float4(__uint_as_float(r[4 * v]) * inv, __uint_as_float(r[4 * v + 1]) * inv,
                            __uint_as_float(r[4 * v + 2]) * inv, __uint_as_float(r[4 * v + 3]) * inv);
        }
      }
      if (valid) {
        const float lse = (l_run > 0.f) ? m_run * p.scale_ln + logf(l_run) : -INFINITY;
        if (kMode == 0) {
          if (p.lse) p.lse[(static_cast<size_t>(b) * Hq + head) * p.geom.L + qrow] = lse;
        } else {
          bool to_sub;
          const size_t r = p2_row(p, w, head, qrow, &to_sub);
          (to_sub ? p.sub_lse : p.part_lse)[r] = lse;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, C::kTmemCols);
}

size_t attn_smem_bytes(int D) {
  return D == 128 ? AttnCfg<128>::kBytes : AttnCfg<64>::kBytes;
}

cudaError_t launch_attn(const AttnParams& p, int D, cudaStream_t stream) {
  if (p.num_items <= 0) return cudaSuccess;
  const size_t smem = attn_smem_bytes(D);
  int dev = 0;
  cudaGetDevice(&dev);
  const bool chunk = p.mode == 1;
  const void* fn = D == 128 ? (chunk ? (const void*)attn_kernel<128, 1> : (const void*)attn_kernel<128, 0>)
                            : (chunk ? (const void*)attn_kernel<64, 1> : (const void*)attn_kernel<64, 0>);
  cudaError_t ea = set_smem_attr_once(fn, (D == 128 ? 2 : 0) + (chunk ? 1 : 0), dev, smem);
  if (ea != cudaSuccess) return ea;
  if (D == 128 && chunk)
    attn_kernel<128, 1><<<p.num_items, kAttnThreads, smem, stream>>>(p);
  else if (D == 128)
    attn_kernel<128, 0><<<p.num_items, kAttnThreads, smem, stream>>>(p);
  else if (chunk)
    attn_kernel<64, 1><<<p.num_items, kAttnThreads, smem, stream>>>(p);
  else
    attn_kernel<64, 0><<<p.num_items, kAttnThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace star
