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
//  * A split is cut into chunks of `chunk` keys, one CTA each, so that the
//    grid covers all 148 SMs even when (batch x KV heads x blocks) is small.
//    CTAs reduce their chunk in-kernel; the last CTA to finish a chunk of a
//    split combines that split's chunks in fixed order (deterministic).
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

#include "star_common.cuh"
#include "star_kernels.cuh"

namespace star {

namespace {

constexpr int kDecStages = 3;
constexpr int kDecThreads = 160;  // 4 consumer warps + 1 producer warp

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

// Reduce the chunk partials of one split (fixed order) into part_o /
// part_lse. Run by the last CTA that finished a chunk of the split; `sw` is
// free shared memory (>= kDecRows * (kMaxChunksPerSplit + 2) floats).
template <int D>
__device__ void reduce_split(const DecodeParams& p, int bh, int split, float* sw) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nwarps = blockDim.x / 32;
  const int nsplit = p.n + 1;
  int first, count;
  if (split < p.n - 1) {
    first = split * p.nc_full;
    count = p.nc_full;
  } else if (split == p.n - 1) {
    first = (p.n - 1) * p.nc_full;
    count = p.nc_last;
  } else {
    first = (p.n - 1) * p.nc_full + p.nc_last;
    count = p.nc_tail;
  }
  const size_t cbase = static_cast<size_t>(bh) * p.chunks_per_head + first;
  float* wgt = sw;                          // [R][count] weights exp(lse_c - M)
  float* rowz = sw + kDecRows * kMaxChunksPerSplit;  // [R] sum of weights
  float* rowm = rowz + kDecRows;            // [R] max statistic
  for (int rho = warp; rho < p.R; rho += nwarps) {
    float M = -INFINITY;
    for (int c = lane; c < count; c += 32) M = fmaxf(M, p.ws_lse[(cbase + c) * kDecRows + rho]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float z = 0.f;
    for (int c = lane; c < count; c += 32) {
      const float l = p.ws_lse[(cbase + c) * kDecRows + rho];
      const float wv = (M == -INFINITY || l == -INFINITY) ? 0.f : expf(l - M);
      wgt[rho * kMaxChunksPerSplit + c] = wv;
      z += wv;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane == 0) {
      rowz[rho] = z;
      rowm[rho] = M;
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < p.R * D; idx += blockDim.x) {
    const int rho = idx / D, d = idx % D;
    float acc = 0.f;
    for (int c = 0; c < count; ++c)  // independent loads: the weights are known
      acc += wgt[rho * kMaxChunksPerSplit + c] * p.ws_o[((cbase + c) * kDecRows + rho) * D + d];
    const float z = rowz[rho];
    const int t = rho / p.g, h = (bh % p.Hkv) * p.g + rho % p.g;
    const int b = bh / p.Hkv;
    const size_t row = ((static_cast<size_t>(b) * p.Hq + h) * nsplit + split) * p.T + t;
    p.part_o[row * D + d] = (z > 0.f) ? acc / z : 0.f;
    if (d == 0) p.part_lse[row] = (z > 0.f) ? rowm[rho] + logf(z) : -INFINITY;
  }
}

template <int D>
__global__ void __launch_bounds__(kDecThreads, 2) decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int kHalfBytes = kDecTile * 128;        // one 64-column TMA box of a tile
  constexpr int kTileBytes = kHalfBytes * (D / 64);  // K (or V) tile of 64 keys
  constexpr int kKSteps = D / 16;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* sK = sm;
  uint8_t* sV = sm + kDecStages * kTileBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + 2 * kDecStages * kTileBytes);
  uint64_t* empty = full + kDecStages;
  __shared__ volatile int abort_flag;
  __shared__ int issued;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int unit = blockIdx.x;
  const int bh = unit / p.chunks_per_head;  // b * Hkv + kvh
  const int cidx = unit % p.chunks_per_head;
  const int b = bh / p.Hkv, kvh = bh % p.Hkv;
  const ChunkRange cr = chunk_range(p, cidx);
  const int ntiles = ceil_div(cr.k_hi - cr.k_lo, kDecTile);

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

  // per-thread softmax state (consumer warps)
  float o[D / 8][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int gq = lane >> 2, t4 = lane & 3;
  const int r0 = gq, r1 = gq + 8;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&p.tmK);
      prefetch_tmap(&p.tmV);
      int it = 0;
      for (; it < ntiles; ++it) {
        const int st = it % kDecStages, use = it / kDecStages;
        if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, &abort_flag, p.status)) break;
        const int key0 = cr.k_lo + it * kDecTile;
        mbar_arrive_expect_tx(&full[st], 2 * kTileBytes);
#pragma unroll
        for (int hd = 0; hd < D / 64; ++hd) {
          tma_load_3d(sK + st * kTileBytes + hd * kHalfBytes, &p.tmK, &full[st], hd * 64, key0, bh);
          tma_load_3d(sV + st * kTileBytes + hd * kHalfBytes, &p.tmV, &full[st], hd * 64, key0, bh);
        }
      }
      issued = it;
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int g = p.g;
    // rows rho = t * g + hh of this GQA group; rows >= R are zero padding
    auto qrow = [&](int rho) -> const __nv_bfloat16* {
      if (rho >= p.R) return nullptr;
      int t = rho / g, hh = rho % g;
      return p.q + ((static_cast<size_t>(b) * p.T + t) * p.Hq + kvh * g + hh) * D;
    };
    const __nv_bfloat16* q0 = qrow(r0);
    const __nv_bfloat16* q1 = qrow(r1);
    uint32_t qf[kKSteps][4];
#pragma unroll
    for (int kk = 0; kk < kKSteps; ++kk) {
      const int c0 = 16 * kk + 2 * t4;
      qf[kk][0] = q0 ? *reinterpret_cast<const uint32_t*>(q0 + c0) : 0u;
      qf[kk][1] = q1 ? *reinterpret_cast<const uint32_t*>(q1 + c0) : 0u;
      qf[kk][2] = q0 ? *reinterpret_cast<const uint32_t*>(q0 + c0 + 8) : 0u;
      qf[kk][3] = q1 ? *reinterpret_cast<const uint32_t*>(q1 + c0 + 8) : 0u;
    }
#pragma unroll
    for (int dn = 0; dn < D / 8; ++dn) o[dn][0] = o[dn][1] = o[dn][2] = o[dn][3] = 0.f;
    const int pos0 = p.L + p.tail_len + r0 / g;  // query positions of this thread's rows
    const int pos1 = p.L + p.tail_len + r1 / g;
    const float c = p.scale_log2;

    for (int it = 0; it < ntiles; ++it) {
      const int st = it % kDecStages;
      if (!mbar_wait(&full[st], (it / kDecStages) & 1, &abort_flag, p.status)) break;
      const uint32_t kb = smem_u32(sK + st * kTileBytes);
      const uint32_t vb = smem_u32(sV + st * kTileBytes);

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
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int key = kbase + 8 * nt + (j & 1);
          const int pos = (j < 2) ? pos0 : pos1;
          const bool vis = key < cr.k_hi && (!cr.causal || key <= pos);
          if (!vis) s[nt][j] = -INFINITY;
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
      for (int nt = 0; nt < 2; ++nt) {
        pr[nt][0] = ex2_approx(fmaf(s[nt][0], c, -ref0));
        pr[nt][1] = ex2_approx(fmaf(s[nt][1], c, -ref0));
        pr[nt][2] = ex2_approx(fmaf(s[nt][2], c, -ref1));
        pr[nt][3] = ex2_approx(fmaf(s[nt][3], c, -ref1));
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
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  }

  // Drain: make sure no TMA copy still targets this CTA's shared memory.
  __syncthreads();
  if (threadIdx.x == 128 && abort_flag) {
    for (int it = imax(0, issued - kDecStages); it < issued; ++it)
      mbar_drain(&full[it % kDecStages], (it / kDecStages) & 1, 100000000ull);
  }
  __syncthreads();
  if (abort_flag) return;

  // Combine the 4 warps' partials through shared memory (the ring is free).
  float* cm = reinterpret_cast<float*>(sm);  // [4][16]
  float* cl = cm + 4 * kDecRows;             // [4][16]
  float* co = cl + 4 * kDecRows;             // [4][16][D]
  if (warp < 4) {
    if (t4 == 0) {
      cm[warp * kDecRows + r0] = m0;
      cm[warp * kDecRows + r1] = m1;
      cl[warp * kDecRows + r0] = l0;
      cl[warp * kDecRows + r1] = l1;
    }
#pragma unroll
    for (int dn = 0; dn < D / 8; ++dn) {
      const int d = 8 * dn + 2 * t4;
      co[(warp * kDecRows + r0) * D + d] = o[dn][0];
      co[(warp * kDecRows + r0) * D + d + 1] = o[dn][1];
      co[(warp * kDecRows + r1) * D + d] = o[dn][2];
      co[(warp * kDecRows + r1) * D + d + 1] = o[dn][3];
    }
  }
  __syncthreads();
  const size_t base = static_cast<size_t>(bh) * p.chunks_per_head + cidx;
  for (int idx = threadIdx.x; idx < p.R * D; idx += blockDim.x) {
    const int rho = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, cm[w * kDecRows + rho]);
    float out = 0.f, lse = -INFINITY;
    if (M != -INFINITY) {
      float Ls = 0.f, acc = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float e = ex2_approx((cm[w * kDecRows + rho] - M) * p.scale_log2);
        Ls += e * cl[w * kDecRows + rho];
        acc += e * co[(w * kDecRows + rho) * D + d];
      }
      out = acc / Ls;
      lse = M * p.scale_ln + logf(Ls);
    }
    p.ws_o[(base * kDecRows + rho) * D + d] = out;
    if (d == 0) p.ws_lse[base * kDecRows + rho] = lse;
  }
  // The last CTA to finish a chunk of this split reduces the split: every
  // CTA publishes its partial (fence) before counting itself in.
  __shared__ int is_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(&p.counters[bh * (p.n + 1) + cr.split], 1);
    const int in_split = cr.split < p.n - 1 ? p.nc_full : (cr.split == p.n - 1 ? p.nc_last : p.nc_tail);
    is_last = (prev == in_split - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  reduce_split<D>(p, bh, cr.split, reinterpret_cast<float*>(sm));
}

size_t decode_smem_bytes(int D) {
  const size_t tile = static_cast<size_t>(kDecTile) * D * 2;
  return 1024 + 2 * kDecStages * tile + 2 * kDecStages * sizeof(uint64_t);
}

cudaError_t launch_decode(const DecodeParams& p, int D, cudaStream_t stream) {
  const int units = p.B * p.Hkv * p.chunks_per_head;
  const size_t smem = decode_smem_bytes(D);
  int dev = 0;
  cudaGetDevice(&dev);
  static bool attr128[64] = {}, attr64[64] = {};
  bool* attr = (D == 128) ? attr128 : attr64;
  if (dev >= 64 || !attr[dev]) {
    cudaError_t e = cudaFuncSetAttribute(D == 128 ? decode_kernel<128> : decode_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if (dev < 64) attr[dev] = true;
  }
  if (D == 128)
    decode_kernel<128><<<units, kDecThreads, smem, stream>>>(p);
  else
    decode_kernel<64><<<units, kDecThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace star
