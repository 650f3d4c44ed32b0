// Phase 2 decode: split-KV attention of a few new tokens over the whole
// cache, one split per context block plus the tail, emitting a
// softmax-normalised partial output and its LSE per split
// [pith 2WVXFXZ2, Referee summary: each host computes local softmax
// statistics over its own KV; abstract: response tokens attend to all prior
// cached tokens].
//
// HBM-bound: every step streams the whole K/V cache once. Design:
//  * The T*g (token, query-head) rows of one GQA group form one 16-row tile,
//    so each K/V byte is read once for all g heads of its group.
//  * A split is cut into chunks of `chunk` keys; the (head, chunk) units are
//    spread over a persistent grid of two CTAs per SM, each streaming a
//    contiguous run of units without a pause between them. A CTA reduces
//    each chunk in-kernel; the CTA completing a split's last chunk combines
//    that split's chunks in fixed order (deterministic), and the CTA
//    completing a head's last split merges the splits when asked to.
//  * A producer warp streams 64-key K/V tiles with TMA (128-byte swizzle)
//    into a 3-stage shared-memory ring; four consumer warps each own 16 keys
//    of a tile.
//  * With g = 8 query heads per KV head a key costs 2*g*D = 2048 multiply-
//    adds: on CUDA cores that alone would need ~70% of the fp32 issue rate at
//    full HBM bandwidth, so the two small products (Q K^T and P V) run on
//    mma.sync m16n8k16 bf16 -> fp32 while the data movement stays TMA.
//  * Softmax statistics are reduced across the 4 lanes of a row quad with
//    warp shuffles; per-warp partials are combined through shared memory.
#include <math.h>

#include "rope_math.cuh"
#include "star_common.cuh"
#include "star_kernels.cuh"

namespace star {

namespace {

constexpr int kDecStages = 3;
constexpr int kDecThreads = 160;  // 4 consumer warps + 1 producer warp
constexpr int kTabPairs = 256;    // (token, frequency) cos/sin pairs per table round

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Bounded wait that ignores the abort flag (used to drain copies in flight).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > limit_ns) return;
  }
}

struct ChunkRange {
  int split, k_lo, k_hi, causal;
};

__device__ __forceinline__ ChunkRange chunk_range(const DecodeParams& p, int c) {
  ChunkRange r;
  int n1 = (p.n - 1) * p.nc_full;
  int cc;
  if (c < n1) {
    r.split = c / p.nc_full;
    cc = c % p.nc_full;
  } else if (c < n1 + p.nc_last) {
    r.split = p.n - 1;
    cc = c - n1;
  } else {
    r.split = p.n;
    cc = c - n1 - p.nc_last;
  }
  int lo, hi;
  if (r.split < p.n) {
    lo = r.split * p.b;
    hi = imin(lo + p.b, p.L);
    r.causal = 0;
  } else {
    lo = p.L;
    hi = p.L + p.tail_len + p.T;
    r.causal = 1;
  }
  r.k_lo = lo + cc * p.chunk;
  r.k_hi = imin(r.k_lo + p.chunk, hi);
  return r;
}

}  // namespace

constexpr int kConsumers = 128;  // threads of the four consumer warps

// Barrier among the four consumer warps only (the producer warp runs ahead).
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}
// Consumer barrier that also returns whether any consumer thread passed a
// non-zero flag: every consumer warp takes the same branch afterwards.
__device__ __forceinline__ bool consumer_sync_or(int flag) {
  uint32_t any;
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.s32 p, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 128, p;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(any)
      : "r"(flag)
      : "memory");
  return any != 0;
}

__device__ __forceinline__ void split_chunks(const DecodeParams& p, int split, int* first,
                                             int* count) {
  if (split < p.n - 1) {
    *first = split * p.nc_full;
    *count = p.nc_full;
  } else if (split == p.n - 1) {
    *first = (p.n - 1) * p.nc_full;
    *count = p.nc_last;
  } else {
    *first = (p.n - 1) * p.nc_full + p.nc_last;
    *count = p.nc_tail;
  }
}

// Weighted LSE combine of `count` partials (lse l_j, normalised rows o_j) of
// one row, four columns at a time: o = sum_j w_j o_j / sum_j w_j, lse = M +
// log sum_j w_j with w_j = e^(l_j - M), M = max_j l_j. The partials are read
// in batches of kBatch with all loads of a batch issued together, the max
// taken in registers (one round trip per batch, no shared memory); a later
// batch with a larger max rescales the running sums.
template <int kBatch, typename LseAt, typename OAt>
__device__ __forceinline__ float4 lse_combine(int count, LseAt lse_at, OAt o_at, float* lse_out) {
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float z = 0.f, M = -INFINITY;
  for (int c0 = 0; c0 < count; c0 += kBatch) {
    float l[kBatch];
    float4 v[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const bool in = c0 + j < count;
      l[j] = in ? lse_at(c0 + j) : -INFINITY;
      v[j] = in ? o_at(c0 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mb = M;
#pragma unroll
    for (int j = 0; j < kBatch; ++j) mb = fmaxf(mb, l[j]);
    if (mb == -INFINITY) continue;
    if (mb > M) {
      const float a = (M == -INFINITY) ? 0.f : expf(M - mb);
      acc = make_float4(acc.x * a, acc.y * a, acc.z * a, acc.w * a);
      z *= a;
      M = mb;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const float w = (l[j] == -INFINITY) ? 0.f : expf(l[j] - M);
      acc = make_float4(acc.x + w * v[j].x, acc.y + w * v[j].y, acc.z + w * v[j].z,
                        acc.w + w * v[j].w);
      z += w;
    }
  }
  const float inv = (z > 0.f) ? 1.f / z : 0.f;
  *lse_out = (z > 0.f) ? M + logf(z) : -INFINITY;
  return make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

// Reduce the chunk partials of one split (fixed order) into part_o /
// part_lse. Run by the consumer warps of the CTA that finished the split's
// last chunk; each thread owns (row, 4 columns) items.
template <int D>
__device__ void reduce_split(const DecodeParams& p, int bh, int split) {
  int first, count;
  split_chunks(p, split, &first, &count);
  const size_t cbase = static_cast<size_t>(bh) * p.chunks_per_head + first;
  const int b = bh / p.Hkv;
  for (int idx = threadIdx.x; idx < p.R * (D / 4); idx += kConsumers) {
    const int rho = idx / (D / 4), d4 = idx % (D / 4);
    float lse;
    const float4 o = lse_combine<16>(
        count, [&](int c) { return p.ws_lse[(cbase + c) * kDecRows + rho]; },
        [&](int c) { return reinterpret_cast<const float4*>(p.ws_o + ((cbase + c) * kDecRows + rho) * D)[d4]; },
        &lse);
    const int t = rho / p.g, h = (bh % p.Hkv) * p.g + rho % p.g;
    const size_t row = ((static_cast<size_t>(b) * p.Hq + h) * p.nsplit + split) * p.T + t;
    reinterpret_cast<float4*>(p.part_o + row * D)[d4] = o;
    if (d4 == 0) p.part_lse[row] = lse;
  }
}

// Exact LSE merge of the split partials of one (batch, KV head) into
// o_merged / lse_merged: m = max lse_s, w_s = exp(lse_s - m),
// o = sum w_s o_s / sum w_s, lse = m + log(sum w_s) [pith 2WVXFXZ2, minor
// comment on Algorithm 2]. Consumer warps only.
template <int D>
__device__ void merge_head(const DecodeParams& p, int bh) {
  const int b = bh / p.Hkv, kvh = bh % p.Hkv;
  for (int idx = threadIdx.x; idx < p.R * (D / 4); idx += kConsumers) {
    const int rho = idx / (D / 4), d4 = idx % (D / 4);
    const int t = rho / p.g, h = kvh * p.g + rho % p.g;
    const size_t row0 = (static_cast<size_t>(b) * p.Hq + h) * p.nsplit;
    float lse;
    const float4 o = lse_combine<8>(
        p.nsplit, [&](int sp) { return p.part_lse[(row0 + sp) * p.T + t]; },
        [&](int sp) { return reinterpret_cast<const float4*>(p.part_o + ((row0 + sp) * p.T + t) * D)[d4]; },
        &lse);
    __nv_bfloat16* dst = p.o_merged + ((static_cast<size_t>(b) * p.T + t) * p.Hq + h) * D + 4 * d4;
    uint2 pk;
    pk.x = pack_bf16x2(o.x, o.y);
    pk.y = pack_bf16x2(o.z, o.w);
    *reinterpret_cast<uint2*>(dst) = pk;
    if (d4 == 0 && p.lse_merged) p.lse_merged[(static_cast<size_t>(b) * p.Hq + h) * p.T + t] = lse;
  }
}

// Combine of the four consumer warps' partials of one unit (rows r0/r1 of
// this lane, 16 keys per warp) into the chunk partial (ws_o, ws_lse). The
// row statistics are exchanged first (cm, cl: [4][kDecRows]); each warp then
// scales its own output by e^(m_w - M) / L (M the row max, L the combined
// row sum), so the output columns are plain 4-term sums, kCols per round
// through `co` ([4][kDecRows][kCols] floats), in a fixed order.
template <int D, int kCols>
__device__ __forceinline__ void combine_warps(const DecodeParams& p, float (&o)[D / 8][4],
                                              float m0, float m1, float l0, float l1, float* cm,
                                              float* cl, float* co, size_t base) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t4 = lane & 3, r0 = lane >> 2, r1 = r0 + 8;
  const float c = p.scale_log2;
  if (t4 == 0) {
    cm[warp * kDecRows + r0] = m0;
    cm[warp * kDecRows + r1] = m1;
    cl[warp * kDecRows + r0] = l0;
    cl[warp * kDecRows + r1] = l1;
  }
  consumer_sync();
  float sc[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int rho = k ? r1 : r0;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, cm[w * kDecRows + rho]);
    float Ls = 0.f, mine = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float e = ex2_approx((cm[w * kDecRows + rho] - M) * c);
        Ls += e * cl[w * kDecRows + rho];
        if (w == warp) mine = e;
      }
    }
    sc[k] = (Ls > 0.f) ? mine / Ls : 0.f;
    if (warp == 0 && t4 == 0 && rho < p.R)
      p.ws_lse[base * kDecRows + rho] = (Ls > 0.f) ? M * p.scale_ln + logf(Ls) : -INFINITY;
  }
#pragma unroll
  for (int dn = 0; dn < D / 8; ++dn) {
    o[dn][0] *= sc[0];
    o[dn][1] *= sc[0];
    o[dn][2] *= sc[1];
    o[dn][3] *= sc[1];
  }
#pragma unroll
  for (int rd = 0; rd < D / kCols; ++rd) {
#pragma unroll
    for (int dn = rd * (kCols / 8); dn < (rd + 1) * (kCols / 8); ++dn) {
      const int d = 8 * dn + 2 * t4 - rd * kCols;
      co[(warp * kDecRows + r0) * kCols + d] = o[dn][0];
      co[(warp * kDecRows + r0) * kCols + d + 1] = o[dn][1];
      co[(warp * kDecRows + r1) * kCols + d] = o[dn][2];
      co[(warp * kDecRows + r1) * kCols + d + 1] = o[dn][3];
    }
    consumer_sync();
    for (int idx = threadIdx.x; idx < p.R * kCols; idx += kConsumers) {
      const int rho = idx / kCols, dc = idx % kCols;
      float out = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) out += co[(w * kDecRows + rho) * kCols + dc];
      p.ws_o[(base * kDecRows + rho) * D + rd * kCols + dc] = out;
    }
    consumer_sync();
  }
}

// Persistent split-KV decode. CTA c owns the contiguous unit range
// [c*U/G, (c+1)*U/G) of the U = B*Hkv*chunks_per_head (head, chunk) units.
// The producer warp streams every tile of every unit through one ring; the
// consumers keep the running softmax of a unit in registers, combine the four
// warps through shared memory at its end, publish the chunk partial, and the
// CTA completing a split (or a head) reduces (merges) it while the producer
// already streams the next unit.
template <int D>
__global__ void __launch_bounds__(kDecThreads, 2) decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int kHalfBytes = kDecTile * 128;        // one 64-column TMA box of a tile
  constexpr int kTileBytes = kHalfBytes * (D / 64);  // K (or V) tile of 64 keys
  constexpr int kKSteps = D / 16;
  constexpr int kCombCols = 32;                      // columns combined per round

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* sK = sm;
  uint8_t* sV = sm + kDecStages * kTileBytes;
  float* comb = reinterpret_cast<float*>(sm + 2 * kDecStages * kTileBytes);  // combine buffer
  float* cm = comb;                                  // [4][16] warp maxima
  float* cl = cm + 4 * kDecRows;                     // [4][16] warp sums
  float* co = cl + 4 * kDecRows;                     // [4][16][kCombCols] warp outputs
  uint64_t* full = reinterpret_cast<uint64_t*>(co + 4 * kDecRows * kCombCols);
  uint64_t* empty = full + kDecStages;
  __shared__ volatile int abort_flag;
  __shared__ int issued;
  __shared__ int flag_last;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int units = p.B * p.Hkv * p.chunks_per_head;
  const int u_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * units / gridDim.x);
  const int u_end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * units / gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    fence_barrier_init();
    abort_flag = 0;
    issued = 0;
  }
  __syncthreads();
  // the next kernel in the stream may be scheduled as this one's CTAs exit
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&p.tmK);
      prefetch_tmap(&p.tmV);
    }
    // The previous kernel in the stream may still be running (programmatic
    // dependent launch). Cache rows [0, L) are written only by Phase 1,
    // whose kernels never start a dependent early and are always followed by
    // another kernel, so tiles of those rows are loaded at once; the tail
    // rows (appended by the previous step) and the append wait for the
    // previous kernel's end.
    bool waited = false;
    const int row0 = p.L + p.tail_len;  // cache row of new token 0
    int gt = 0;  // tiles issued over all units of this CTA
    bool stop = false;
    for (int u = u_begin; u < u_end && !stop; ++u) {
      const int bh = u / p.chunks_per_head;
      const ChunkRange cr = chunk_range(p, u % p.chunks_per_head);
      const int nt = ceil_div(cr.k_hi - cr.k_lo, kDecTile);
      // This call's tokens: the unit whose key range holds a new token's cache
      // row rotates its key and appends key and value before loading that
      // tile (no other unit reads the row). The warp writes, every lane
      // fences its generic writes against the TMA (async proxy) reads.
      const int w_lo = imax(cr.k_lo, row0), w_hi = p.with_tail ? imin(cr.k_hi, row0 + p.T) : 0;
      if (w_lo < w_hi && !waited) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        waited = true;
      }
      if (w_lo < w_hi) {
        const int b = bh / p.Hkv, kvh = bh % p.Hkv;
        for (int r = w_lo; r < w_hi; ++r) {
          const int t = r - row0;
          const __nv_bfloat16* ks = p.k_new + ((static_cast<size_t>(b) * p.T + t) * p.Hkv + kvh) * D;
          const __nv_bfloat16* vs = p.v_new + ((static_cast<size_t>(b) * p.T + t) * p.Hkv + kvh) * D;
          __nv_bfloat16* kd = p.k_cache + (static_cast<size_t>(bh) * p.Lcap + r) * D;
          __nv_bfloat16* vd = p.v_cache + (static_cast<size_t>(bh) * p.Lcap + r) * D;
          for (int i = lane; i < D / 2; i += 32) {
            double c64, s64;
            rope_angle(static_cast<long long>(p.ctx_pos0) + r, p.inv_freq[i], &c64, &s64);
            const float a = __bfloat162float(ks[i]), bb = __bfloat162float(ks[i + D / 2]);
            const float c32 = static_cast<float>(c64), s32 = static_cast<float>(s64);
            kd[i] = __ushort_as_bfloat16(static_cast<unsigned short>(rope_rotate_bf16(a, bb, c32, s32, c64, s64, true)));
            kd[i + D / 2] = __ushort_as_bfloat16(static_cast<unsigned short>(rope_rotate_bf16(a, bb, c32, s32, c64, s64, false)));
          }
          for (int i = lane; i < D; i += 32) vd[i] = vs[i];
        }
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncwarp();
      }
      for (int it = 0; it < nt; ++it, ++gt) {
        if (!waited && cr.k_lo + (it + 1) * kDecTile > p.L) {  // reaches the tail rows
          asm volatile("griddepcontrol.wait;" ::: "memory");
          waited = true;
        }
        int ok = 1;
        if (lane == 0) {
          const int st = gt % kDecStages, use = gt / kDecStages;
          if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, &abort_flag, p.status)) {
            ok = 0;
          } else {
            const int key0 = cr.k_lo + it * kDecTile;
            mbar_arrive_expect_tx(&full[st], 2 * kTileBytes);
#pragma unroll
            for (int hd = 0; hd < D / 64; ++hd) {
              tma_load_3d(sK + st * kTileBytes + hd * kHalfBytes, &p.tmK, &full[st], hd * 64, key0, bh);
              tma_load_3d(sV + st * kTileBytes + hd * kHalfBytes, &p.tmV, &full[st], hd * 64, key0, bh);
            }
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          stop = true;
          break;
        }
      }
    }
    if (lane == 0) {
      issued = gt;  // a failed wait breaks before counting its tile
      if (abort_flag) {  // let copies still in flight land before the CTA exits
        for (int it = imax(0, issued - kDecStages); it < issued; ++it)
          mbar_drain(&full[it % kDecStages], (it / kDecStages) & 1, 100000000ull);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int gq = lane >> 2, t4 = lane & 3;
    const int r0 = gq, r1 = gq + 8;
    const int g = p.g;
    const float c = p.scale_log2;
    uint32_t qf[kKSteps][4];
    int q_bh = -1;
    bool q_waited = false;
    int gt = 0;  // tiles consumed over all units of this CTA
    for (int u = u_begin; u < u_end; ++u) {
      const int bh = u / p.chunks_per_head;
      const int cidx = u % p.chunks_per_head;
      const int b = bh / p.Hkv, kvh = bh % p.Hkv;
      const ChunkRange cr = chunk_range(p, cidx);
      const int nt = ceil_div(cr.k_hi - cr.k_lo, kDecTile);
      if (bh != q_bh) {
        // rows rho = t * g + hh of this GQA group (rows >= R are zero padding):
        // rotate them here (shared RoPE arithmetic, bit-identical to the
        // RoPE kernel) into the free combine buffer, then take fragments.
        // cos/sin (fp64) of each (token, frequency) pair are computed once,
        // kTabPairs at a time, into the buffer after the rows: the g rows of
        // a token share them.
        uint16_t* qs = reinterpret_cast<uint16_t*>(comb);  // [kDecRows][D] bf16 bits
        double* tcos = reinterpret_cast<double*>(qs + kDecRows * D);
        double* tsin = tcos + kTabPairs;
        constexpr int kTabTok = kTabPairs / (D / 2);       // tokens per table round
        for (int e = p.R * (D / 2) + threadIdx.x; e < kDecRows * (D / 2); e += kConsumers) {
          const int rho = e / (D / 2), i = e % (D / 2);
          qs[rho * D + i] = 0;
          qs[rho * D + i + D / 2] = 0;
        }
        for (int t0 = 0; t0 < p.T; t0 += kTabTok) {
          const int tn = imin(kTabTok, p.T - t0);
          for (int e = threadIdx.x; e < tn * (D / 2); e += kConsumers)
            rope_angle(static_cast<long long>(p.q_pos0) + t0 + e / (D / 2),
                       p.inv_freq[e % (D / 2)], &tcos[e], &tsin[e]);
          consumer_sync();
          // q may be written by the kernel just before this one (a projection,
          // or a caller's own kernel that starts its dependents early): read
          // it only after that kernel has ended. The cos/sin table above
          // depends on positions only and is built before the wait.
          if (!q_waited) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            q_waited = true;
          }
          for (int e = threadIdx.x; e < tn * g * (D / 2); e += kConsumers) {
            const int rl = e / (D / 2), i = e % (D / 2);
            const int tl = rl / g, rho = t0 * g + rl;
            const __nv_bfloat16* src =
                p.q_new + ((static_cast<size_t>(b) * p.T + t0 + tl) * p.Hq + kvh * g + rl % g) * D;
            const double c64 = tcos[tl * (D / 2) + i], s64 = tsin[tl * (D / 2) + i];
            const float a = __bfloat162float(src[i]), bb = __bfloat162float(src[i + D / 2]);
            const float c32 = static_cast<float>(c64), s32 = static_cast<float>(s64);
            qs[rho * D + i] = static_cast<uint16_t>(rope_rotate_bf16(a, bb, c32, s32, c64, s64, true));
            qs[rho * D + i + D / 2] =
                static_cast<uint16_t>(rope_rotate_bf16(a, bb, c32, s32, c64, s64, false));
          }
          consumer_sync();  // the table is rewritten by the next round
        }
#pragma unroll
        for (int kk = 0; kk < kKSteps; ++kk) {
          const int c0 = 16 * kk + 2 * t4;
          qf[kk][0] = *reinterpret_cast<const uint32_t*>(qs + r0 * D + c0);
          qf[kk][1] = *reinterpret_cast<const uint32_t*>(qs + r1 * D + c0);
          qf[kk][2] = *reinterpret_cast<const uint32_t*>(qs + r0 * D + c0 + 8);
          qf[kk][3] = *reinterpret_cast<const uint32_t*>(qs + r1 * D + c0 + 8);
        }
        consumer_sync();  // the buffer is reused by the combine below
        q_bh = bh;
      }
      float o[D / 8][4];
#pragma unroll
      for (int dn = 0; dn < D / 8; ++dn) o[dn][0] = o[dn][1] = o[dn][2] = o[dn][3] = 0.f;
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
      const int pos0 = p.L + p.tail_len + r0 / g;  // cache rows of this thread's query tokens
      const int pos1 = p.L + p.tail_len + r1 / g;

      for (int it = 0; it < nt; ++it, ++gt) {
        const int st = gt % kDecStages;
        if (!mbar_wait(&full[st], (gt / kDecStages) & 1, &abort_flag, p.status)) break;
        const uint32_t kb = smem_u32(sK + st * kTileBytes);
        const uint32_t vb = smem_u32(sV + st * kTileBytes);
        // A tile that runs past the unit's last key holds rows of other units
        // (or of this call's new tokens, which another CTA may be writing):
        // masked keys get P = 0, but 0 * NaN would still poison P V, so each
        // warp clears its own V rows past the end. The fence orders these
        // generic writes before the next TMA write into the stage.
        {
          const int first_bad = cr.k_hi - (cr.k_lo + it * kDecTile);
          if (first_bad < kDecTile && 16 * warp + 15 >= first_bad) {
            uint8_t* vt = sV + st * kTileBytes;
            for (int idx = lane; idx < 16 * (D / 64) * 8; idx += 32) {
              const int rr = 16 * warp + idx / ((D / 64) * 8);
              const int rem = idx % ((D / 64) * 8);
              if (rr >= first_bad)
                *reinterpret_cast<uint4*>(vt + (rem / 8) * kHalfBytes + rr * 128 + (rem % 8) * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
          }
        }
        // S = Q K^T for this warp's 16 keys (two n-tiles of 8 keys)
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
          const int key_row = 16 * warp + ((lane >> 4) & 1) * 8 + (lane & 7);
#pragma unroll
          for (int kk = 0; kk < kKSteps; ++kk) {
            const int chunk = 2 * kk + ((lane >> 3) & 1);
            const uint32_t addr = kb + (chunk >> 3) * kHalfBytes + sw128_offset(key_row, chunk & 7);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(addr, b0, b1, b2, b3);
            mma_16816(s[0], qf[kk], b0, b1);
            mma_16816(s[1], qf[kk], b2, b3);
          }
        }
        // visibility: keys [k_lo, k_hi) of this chunk, causal in the tail
        const int kbase = cr.k_lo + it * kDecTile + 16 * warp + 2 * t4;
#pragma unroll
        for (int ntl = 0; ntl < 2; ++ntl)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int key = kbase + 8 * ntl + (j & 1);
            const int pos = (j < 2) ? pos0 : pos1;
            const bool vis = key < cr.k_hi && (!cr.causal || key <= pos);
            if (!vis) s[ntl][j] = -INFINITY;
          }
        // online softmax over the two rows this thread touches
        float mt0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
        float mt1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
        mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, 1));
        mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, 2));
        mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, 1));
        mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, 2));
        const float mn0 = fmaxf(m0, mt0), mn1 = fmaxf(m1, mt1);
        const float a0 = (mn0 == -INFINITY) ? 1.f : ex2_approx((m0 - mn0) * c);
        const float a1 = (mn1 == -INFINITY) ? 1.f : ex2_approx((m1 - mn1) * c);
        const float ref0 = (mn0 == -INFINITY) ? 0.f : mn0 * c;
        const float ref1 = (mn1 == -INFINITY) ? 0.f : mn1 * c;
        m0 = mn0;
        m1 = mn1;
        float pr[2][4];
#pragma unroll
        for (int ntl = 0; ntl < 2; ++ntl) {
          pr[ntl][0] = ex2_approx(fmaf(s[ntl][0], c, -ref0));
          pr[ntl][1] = ex2_approx(fmaf(s[ntl][1], c, -ref0));
          pr[ntl][2] = ex2_approx(fmaf(s[ntl][2], c, -ref1));
          pr[ntl][3] = ex2_approx(fmaf(s[ntl][3], c, -ref1));
        }
        l0 = l0 * a0 + (pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1]);
        l1 = l1 * a1 + (pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3]);
#pragma unroll
        for (int dn = 0; dn < D / 8; ++dn) {
          o[dn][0] *= a0;
          o[dn][1] *= a0;
          o[dn][2] *= a1;
          o[dn][3] *= a1;
        }
        uint32_t pa[4];
        pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
        pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
        pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
        pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);
        // O += P V over this warp's 16 keys, two 8-wide d tiles per ldmatrix
        {
          const int mi = lane >> 3;
          const int key_row = 16 * warp + (mi & 1) * 8 + (lane & 7);
#pragma unroll
          for (int dn2 = 0; dn2 < D / 16; ++dn2) {
            const int chunk = 2 * dn2 + (mi >> 1);
            const uint32_t addr = vb + (chunk >> 3) * kHalfBytes + sw128_offset(key_row, chunk & 7);
            uint32_t v0, v1, v2, v3;
            ldsm_x4_t(addr, v0, v1, v2, v3);
            mma_16816(o[2 * dn2], pa, v0, v1);
            mma_16816(o[2 * dn2 + 1], pa, v2, v3);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }
      // all four consumer warps decide together whether to stop (a warp still
      // inside the tile loop would otherwise miss the named barriers below)
      if (consumer_sync_or(abort_flag)) break;
      // the first global write of this call (the previous kernel may still be
      // reducing its own partials from the workspace) follows its end
      asm volatile("griddepcontrol.wait;" ::: "memory");
      if (blockIdx.x == 0 && threadIdx.x == 0 && u == u_begin)
        p.status[1] = p.header_bytes;  // the header this call counts in, for star_device_status
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

      // ---- combine the four warps' partials, kCombCols columns per round
      combine_warps<D, kCombCols>(p, o, m0, m1, l0, l1, cm, cl, co,
                                  static_cast<size_t>(bh) * p.chunks_per_head + cidx);
      // ---- the CTA completing a split reduces it; the one completing a head
      // merges it. After the consumer barrier one thread publishes the CTA's
      // writes (fence, then count itself in) and, if last, fences again so
      // the partials of the other CTAs are visible before anyone reads them.
      consumer_sync();
      if (threadIdx.x == 0) {
        int first, count;
        split_chunks(p, cr.split, &first, &count);
        __threadfence();
        // wraps to 0 on the last arrival: the counter is zero again for the next call
        flag_last = (atomicInc(reinterpret_cast<unsigned*>(&p.counters[bh * p.nsplit + cr.split]),
                               static_cast<unsigned>(count - 1)) == static_cast<unsigned>(count - 1));
        __threadfence();
      }
      consumer_sync();
      if (flag_last) {
        reduce_split<D>(p, bh, cr.split);
        consumer_sync();
        if (p.o_merged != nullptr) {
          if (threadIdx.x == 0) {
            __threadfence();
            flag_last = (atomicInc(reinterpret_cast<unsigned*>(&p.head_counters[bh]),
                                   static_cast<unsigned>(p.nsplit - 1)) ==
                         static_cast<unsigned>(p.nsplit - 1));
            __threadfence();
          }
          consumer_sync();
          if (flag_last) merge_head<D>(p, bh);
          consumer_sync();
        }
      }
    }
  }
  __syncthreads();
}

size_t decode_smem_bytes(int D) {
  const size_t tile = static_cast<size_t>(kDecTile) * D * 2;
  const size_t comb = (2 * 4 * kDecRows + 4 * kDecRows * 32) * sizeof(float);
  return 1024 + 2 * kDecStages * tile + comb + 2 * kDecStages * sizeof(uint64_t);
}

cudaError_t launch_decode(const DecodeParams& p, int D, cudaStream_t stream) {
  const int units = p.B * p.Hkv * p.chunks_per_head;
  const size_t smem = decode_smem_bytes(D);
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t ea = set_smem_attr_once(D == 128 ? (const void*)decode_kernel<128> : (const void*)decode_kernel<64>,
                                      D == 128 ? 9 : 8, dev, smem);
  if (ea != cudaSuccess) return ea;
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = imin(units, 2 * sms);  // persistent: two CTAs per SM
  // programmatic dependent launch: the kernel may start (barriers, tensor
  // maps, the cos/sin table) while the previous kernel in the stream drains;
  // it waits for that kernel's completion before touching global memory
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr_pdl[1];
  attr_pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr_pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr_pdl;
  cfg.numAttrs = 1;
  return (D == 128) ? cudaLaunchKernelEx(&cfg, decode_kernel<128>, p)
                    : cudaLaunchKernelEx(&cfg, decode_kernel<64>, p);
}

}  // namespace star
