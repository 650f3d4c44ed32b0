// Projection GEMMs of the decoder stack on 5th-generation tensor cores
// (tcgen05 + tensor memory + TMA), sm_100a:
//
//   y[M, N] = x[M, K] * w[N, K]^T      bf16 operands, fp32 accumulation
//
// with the epilogues a Star Attention layer needs around its attention
// [pith 2WVXFXZ2, the paper's abstract: the model is unchanged, only
// attention is replaced; "What carries the argument": keys keep their
// original positions]:
//   * plain:     y = bf16(acc)
//   * residual:  y = bf16(y + bf16(acc))  (the stored projection, then the add)
//   * RoPE:      every head of `rd` columns is rotated (rotate-half, pair
//                (i, i + rd/2) turns by pos * theta^(-2i/rd), pos = pos0 +
//                row % seq_len) after the projection is rounded to bf16; the
//                rotation is the library's correctly rounded one, so the bits
//                equal a projection followed by star_rope
//   * cache:     rows go head-major into a KV cache [B, N/rd, cache_rows, rd]
//                (row m = b * seq_len + t lands in cache row t of sequence b),
//                rotated (K) or not (V)
//
// Design: a persistent kernel, one CTA per SM, 320 threads.
//   warp 0     TMA producer: A (128 x 64) and B (256 x 64) tiles, 128-byte
//              swizzle, through a 4-stage shared-memory ring
//   warp 1     TMEM allocator and single-thread tcgen05.mma issuer
//              (M = 128, N = 256, K = 16 per instruction, both operands
//              K-major)
//   warps 2-9  epilogue, two warpgroups: thread = output row = TMEM lane,
//              warps 2-5 take the tile's columns 0-127 and warps 6-9 the
//              columns 128-255 (the RoPE epilogue would otherwise outlast a
//              tile's main loop: one warpgroup left the tensor pipe idle 37%
//              of the time)
// The fp32 accumulator is double-buffered in tensor memory (2 x 256
// columns), so a tile's epilogue overlaps the next tile's MMAs. Tiles are
// taken in row-major order (m outer, n inner), so the CTAs in flight share
// the A rows of one m-tile and every B tile stays in L2.
#include <math.h>

#include "rope_math.cuh"
#include "star_common.cuh"
#include "star_kernels.cuh"

namespace star {

namespace {

constexpr int kGemmThreads = 320;
constexpr int kEpiThreads = 256;  // warps 2-9
constexpr int kBM = 128, kBN = 256, kBK = 64, kGemmStages = 4;
constexpr int kATile = kBM * kBK * 2;  // 16 KB
constexpr int kBTile = kBN * kBK * 2;  // 32 KB
constexpr int kStageBytes = kATile + kBTile;
constexpr int kGemmOffBar = kGemmStages * kStageBytes;
constexpr int kGemmSmem = kGemmOffBar + 256 + 1024;  // + barriers + alignment slack
constexpr uint32_t kAccCols = 256;
constexpr uint64_t kGemmDrainNs = 100000000ull;  // 100 ms

__device__ __forceinline__ void gemm_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > limit_ns) return;
  }
}

__device__ __forceinline__ uint32_t bf16_bits_rn(float x) { return pack_bf16x2(x, 0.f) & 0xFFFFu; }
__device__ __forceinline__ float bf16_round(float x) { return __uint_as_float(bf16_bits_rn(x) << 16); }

// Where one output row goes: element n of row m is at row + n (row-major
// [M, N], cache_rows == 0), or at row + (n / hd) * head_stride + n % hd (the
// head-major cache [B, N / hd, cache_rows, hd]).
struct OutRow {
  __nv_bfloat16* row;
  size_t head_stride;  // 0 for row-major
};
// Output row m of buffer y (width nw columns, in heads of hd for the cache).
__device__ __forceinline__ OutRow out_row(const GemmParams& p, __nv_bfloat16* y, int nw, int m) {
  if (p.cache_rows == 0) return OutRow{y + static_cast<size_t>(m) * nw, 0};
  const int b = m / p.seq_len, t = m - b * p.seq_len;
  const size_t hs = static_cast<size_t>(p.cache_rows) * p.hd;
  return OutRow{y + static_cast<size_t>(b) * (nw / p.hd) * hs + static_cast<size_t>(t) * p.hd, hs};
}
// 8 consecutive columns from n never straddle a head (hd is a multiple of 8)
__device__ __forceinline__ __nv_bfloat16* out_at(const GemmParams& p, const OutRow& o, int n) {
  if (o.head_stride == 0) return o.row + n;
  const int head = n / p.hd;
  return o.row + head * o.head_stride + (n - head * p.hd);
}

// 32 accumulator columns of one row -> bf16 (plus the residual), stored as
// four 16-byte vectors starting at column n (a vector past N is skipped).
__device__ __forceinline__ void store_plain32(const GemmParams& p, const OutRow& o, int n,
                                              const uint32_t (&r)[32]) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    if (n + 8 * v >= p.N) break;
    __nv_bfloat16* dst = out_at(p, o, n + 8 * v);
    uint32_t w[4];
    if (p.accumulate) {
      const uint4 old = *reinterpret_cast<const uint4*>(dst);
      const uint32_t ow[4] = {old.x, old.y, old.z, old.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float a0 = bf16_round(__uint_as_float(r[8 * v + 2 * j])) + bf16_lo(ow[j]);
        const float a1 = bf16_round(__uint_as_float(r[8 * v + 2 * j + 1])) + bf16_hi(ow[j]);
        w[j] = pack_bf16x2(a0, a1);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        w[j] = pack_bf16x2(__uint_as_float(r[8 * v + 2 * j]), __uint_as_float(r[8 * v + 2 * j + 1]));
    }
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// 16 bf16 values (bits in the low 16 of each word) to two 16-byte vectors at column n.
__device__ __forceinline__ void store_bits16(const GemmParams& p, const OutRow& o, int n,
                                             const uint32_t (&h)[16]) {
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    __nv_bfloat16* dst = out_at(p, o, n + 8 * v);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = h[8 * v + 2 * j] | (h[8 * v + 2 * j + 1] << 16);
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// 16 accumulator columns -> bf16, two 16-byte vectors at column n (no residual).
__device__ __forceinline__ void store_plain16(const GemmParams& p, const OutRow& o, int n,
                                              const uint32_t (&r)[16]) {
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    __nv_bfloat16* dst = out_at(p, o, n + 8 * v);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      w[j] = pack_bf16x2(__uint_as_float(r[8 * v + 2 * j]), __uint_as_float(r[8 * v + 2 * j + 1]));
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace

// RD: head dim of the rotated epilogue (64 or 128), 0 for no rotation.
template <int RD>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kGemmOffBar);
  uint64_t* empty = full + kGemmStages;
  uint64_t* acc_full = empty + kGemmStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2]
  uint64_t* done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = p.m_tiles * p.n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&acc_full[x], 1);
      mbar_init(&acc_empty[x], kEpiThreads);
    }
    mbar_init(done, 1);
    fence_barrier_init();
    abort_flag = 0;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * kAccCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&p.tmA);
      prefetch_tmap(&p.tmB);
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x) {
        const int m0 = (tile / p.n_tiles) * kBM, n0 = (tile % p.n_tiles) * kBN;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int st = it % kGemmStages, use = it / kGemmStages;
          if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          uint8_t* a = sm + st * kStageBytes;
          mbar_arrive_expect_tx(&full[st], kStageBytes);
          tma_load_2d(a, &p.tmA, &full[st], kb * kBK, m0);
          tma_load_2d(a + kATile, &p.tmB, &full[st], kb * kBK, n0);
        }
      }
      if (abort_flag) {  // let copies still in flight land before the CTA exits
        for (int j = imax(0, it - kGemmStages); j < it; ++j)
          gemm_drain(&full[j % kGemmStages], (j / kGemmStages) & 1, kGemmDrainNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kBM, kBN, 0, 0);
      const uint32_t base = smem_u32(sm);
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x, ++lt) {
        const int ab = lt & 1, use = lt >> 1;
        if (use > 0 && !mbar_wait(&acc_empty[ab], (use - 1) & 1, &abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t acc = tmem + ab * kAccCols;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int st = it % kGemmStages;
          if (!mbar_wait(&full[st], (it / kGemmStages) & 1, &abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = base + st * kStageBytes, b = a + kATile;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_ss(acc, sdesc_sw128(a + kk * 32, 16, 1024), sdesc_sw128(b + kk * 32, 16, 1024),
                   idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&empty[st]);  // the stage is free once these MMAs have read it
        }
        if (!ok) break;
        mma_commit(&acc_full[ab]);
      }
      // every MMA issued so far (or abandoned) completes before TMEM is freed
      mma_commit(done);
      gemm_drain(done, 0, kGemmDrainNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31 (warps 2-9 -> 2,3,0,1,2,3,0,1)
    const int row = 32 * quad + lane;
    const int half = (warp - 2) >> 2;  // which 128 of the tile's 256 columns
    constexpr int kHalfN = kBN / 2;
    int lt = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++lt) {
      const int ab = lt & 1, use = lt >> 1;
      if (!mbar_wait(&acc_full[ab], use & 1, &abort_flag, p.status)) break;
      tc_fence_after();
      const int m0 = (tile / p.n_tiles) * kBM, n0 = (tile % p.n_tiles) * kBN;
      const int m = m0 + row;
      const bool mvalid = m < p.M;
      const OutRow orow = out_row(p, p.y, p.n_split, mvalid ? m : 0);
      const OutRow orow2 = out_row(p, p.y2, p.N - p.n_split, mvalid ? m : 0);
      const uint32_t tb = tmem + (static_cast<uint32_t>(32 * quad) << 16) + ab * kAccCols;
      if constexpr (RD == 0) {
#pragma unroll 1
        for (int c = half * (kHalfN / 32); c < (half + 1) * (kHalfN / 32); ++c) {
          uint32_t r[32];
          tmem_ld32(tb + 32 * c, r);
          tmem_wait_ld();
          reg_fence32(r);
          if (mvalid && n0 + 32 * c < p.N) store_plain32(p, orow, n0 + 32 * c, r);
        }
      } else {
        // heads of RD columns; pair (i, i + RD/2); 16 frequencies at a time,
        // their fp32 cos/sin read once from the call's table (built by
        // rope_table_kernel) and shared by this warpgroup's heads
        const int t = mvalid ? m % p.seq_len : 0;
        const long long pos = p.pos0 + t;
#pragma unroll 1
        for (int fc = 0; fc < RD / 32; ++fc) {
          float c32[16], s32[16];
          const float4* tab = reinterpret_cast<const float4*>(p.rope_tab + static_cast<size_t>(t) * (RD / 2) + 16 * fc);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 cs = tab[j];
            c32[2 * j] = cs.x;
            s32[2 * j] = cs.y;
            c32[2 * j + 1] = cs.z;
            s32[2 * j + 1] = cs.w;
          }
#pragma unroll 1
          for (int h = half * (kHalfN / RD); h < (half + 1) * (kHalfN / RD); ++h) {
            const int col = h * RD + 16 * fc;  // first-half column of this chunk
            if (n0 + h * RD >= p.N) break;     // warp-uniform
            uint32_t x[16], y[16];
            tmem_ld16(tb + col, x);
            tmem_ld16(tb + col + RD / 2, y);
            tmem_wait_ld();
            reg_fence16(x);
            reg_fence16(y);
            if (n0 + h * RD >= p.n_split) {  // a V head of a K/V projection: no rotation
              if (mvalid) {
                store_plain16(p, orow2, n0 + col - p.n_split, x);
                store_plain16(p, orow2, n0 + col + RD / 2 - p.n_split, y);
              }
              continue;
            }
            if (mvalid) {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                // the stored (bf16) projection is what gets rotated
                const float a = bf16_round(__uint_as_float(x[j]));
                const float b = bf16_round(__uint_as_float(y[j]));
                const uint32_t pr = rope_rotate_pair_bf16_at(a, b, c32[j], s32[j], pos,
                                                             p.inv_freq[16 * fc + j]);
                x[j] = pr & 0xFFFFu;
                y[j] = pr >> 16;
              }
              store_bits16(p, orow, n0 + col, x);
              store_bits16(p, orow, n0 + col + RD / 2, y);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 2 * kAccCols);
}

__global__ void rope_table_kernel(float2* __restrict__ tab, int S, int half, long long pos0,
                                  const __grid_constant__ GemmParams p) {
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= static_cast<long long>(S) * half) return;
  const int t = static_cast<int>(e / half), i = static_cast<int>(e % half);
  double c, s;
  rope_angle(pos0 + t, p.inv_freq[i], &c, &s);
  tab[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

cudaError_t launch_rope_table(float2* tab, int S, int half, long long pos0, const double* inv_freq,
                              cudaStream_t stream) {
  GemmParams p;  // only its frequency table is read
  for (int i = 0; i < 64; ++i) p.inv_freq[i] = inv_freq[i];
  const long long n = static_cast<long long>(S) * half;
  if (n == 0) return cudaSuccess;
  rope_table_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(tab, S, half, pos0, p);
  return cudaGetLastError();
}

size_t gemm_smem_bytes() { return kGemmSmem; }

cudaError_t launch_gemm(const GemmParams& p, int sms, cudaStream_t stream) {
  const int tiles = p.m_tiles * p.n_tiles;
  if (tiles <= 0) return cudaSuccess;
  int dev = 0;
  cudaGetDevice(&dev);
  const void* fn = p.rd == 128 ? (const void*)gemm_kernel<128>
                   : p.rd == 64 ? (const void*)gemm_kernel<64>
                                : (const void*)gemm_kernel<0>;
  const int slot = 4 + (p.rd == 128 ? 2 : p.rd == 64 ? 1 : 0);
  cudaError_t e = set_smem_attr_once(fn, slot, dev, kGemmSmem);
  if (e != cudaSuccess) return e;
  const int grid = imin(tiles, sms);
  if (p.rd == 128)
    gemm_kernel<128><<<grid, kGemmThreads, kGemmSmem, stream>>>(p);
  else if (p.rd == 64)
    gemm_kernel<64><<<grid, kGemmThreads, kGemmSmem, stream>>>(p);
  else
    gemm_kernel<0><<<grid, kGemmThreads, kGemmSmem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace star
