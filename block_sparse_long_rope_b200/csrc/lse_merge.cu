// Exact merge of per-split partials into global attention.
//
// Each split h carries a softmax-normalised output o_h and its log-sum-exp
// lse_h. The pages' corrected online-softmax update weights a split by
// exp(s_h - s_global) [pith 2WVXFXZ2, minor comment on Algorithm 2]; with
// m = max_h lse_h this is
//   w_h = exp(lse_h - m),  o = sum_h w_h o_h / sum_h w_h,  lse = m + log(sum_h w_h)
// which reproduces softmax over the concatenated keys exactly [pith 2WVXFXZ2,
// assumptions: online softmax aggregation yields the exact global softmax].
//
// The splits may come in segments, one per rank after an all-gather of the
// ranks' partials: segment s occupies B * Hq * slots split rows and begins
// with its segs.ns[s] splits laid out [B, Hq, ns[s], T, D]. One segment with
// slots = ns[0] = nsplit is the plain [B, Hq, nsplit, T, D] layout.
//
// One warp per (batch, head, token) row; lanes cover D with 16-byte loads.
// HBM-bound and tiny: it reads nsplit * (D + 1) floats per row.
#include <math.h>

#include "star_common.cuh"
#include "star_kernels.cuh"

namespace star {

template <int D>
__global__ void __launch_bounds__(256) lse_merge_kernel(const float* __restrict__ part_o,
                                                        const float* __restrict__ part_lse,
                                                        const __grid_constant__ MergeSegs segs,
                                                        __nv_bfloat16* __restrict__ o,
                                                        float* __restrict__ lse, int B, int T,
                                                        int Hq) {
  constexpr int kPer = D / 32;  // floats per lane (2 or 4)
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  const int rows = B * Hq * T;
  if (warp >= rows) return;
  const int t = warp % T;
  const int h = (warp / T) % Hq;
  const int b = warp / (T * Hq);
  const size_t bh = static_cast<size_t>(b) * Hq + h;
  const size_t seg_rows = static_cast<size_t>(B) * Hq * segs.slots;  // (b, h, split) rows per segment
  auto split_row = [&](int seg, int s) { return (seg * seg_rows + bh * segs.ns[seg] + s) * T + t; };

  // statistics: lanes read the split LSEs in parallel, shuffles reduce them
  float m = -INFINITY;
  for (int seg = 0; seg < segs.nseg; ++seg)
    for (int s = lane; s < segs.ns[seg]; s += 32) m = fmaxf(m, part_lse[split_row(seg, s)]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float acc[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) acc[j] = 0.f;
  float z = 0.f;
  if (m != -INFINITY) {
    for (int seg = 0; seg < segs.nseg; ++seg) {
      const int nsplit = segs.ns[seg];
      for (int s0 = 0; s0 < nsplit; s0 += 32) {
        const int sl = s0 + lane;
        const float l = (sl < nsplit) ? part_lse[split_row(seg, sl)] : -INFINITY;
        const float wl = (l == -INFINITY) ? 0.f : expf(l - m);
        float zs = wl;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, off);
        z += zs;
        const int ns = imin(32, nsplit - s0);
#pragma unroll 4
        for (int k = 0; k < ns; ++k) {  // independent loads: the weights are already known
          const float w = __shfl_sync(0xffffffffu, wl, k);
          const float* src = part_o + split_row(seg, s0 + k) * D + lane * kPer;
          if constexpr (kPer == 4) {
            const float4 v = *reinterpret_cast<const float4*>(src);
            acc[0] += w * v.x;
            acc[1] += w * v.y;
            acc[2] += w * v.z;
            acc[3] += w * v.w;
          } else {
            const float2 v = *reinterpret_cast<const float2*>(src);
            acc[0] += w * v.x;
            acc[1] += w * v.y;
          }
        }
      }
    }
  }
  const float inv = (z > 0.f) ? 1.f / z : 0.f;
  __nv_bfloat16* dst = o + ((static_cast<size_t>(b) * T + t) * Hq + h) * D + lane * kPer;
  if constexpr (kPer == 4) {
    uint2 pk;
    pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(dst) = pk;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
  if (lse != nullptr && lane == 0) lse[bh * T + t] = (z > 0.f) ? m + logf(z) : -INFINITY;
}

cudaError_t launch_lse_merge(const float* part_o, const float* part_lse, const MergeSegs& segs,
                             __nv_bfloat16* o, float* lse, int B, int T, int Hq, int D,
                             cudaStream_t stream) {
  const long long rows = static_cast<long long>(B) * Hq * T;
  if (rows == 0) return cudaSuccess;
  const int threads = 256;
  const unsigned blocks = static_cast<unsigned>((rows * 32 + threads - 1) / threads);
  if (D == 128)
    lse_merge_kernel<128><<<blocks, threads, 0, stream>>>(part_o, part_lse, segs, o, lse, B, T, Hq);
  else
    lse_merge_kernel<64><<<blocks, threads, 0, stream>>>(part_o, part_lse, segs, o, lse, B, T, Hq);
  return cudaGetLastError();
}

// Device evaluation of the Phase-1 index math for every context row.
__global__ void debug_index_kernel(int L, int b, int a, int32_t* blk, int32_t* pos,
                                   int32_t* ranges) {
  int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= L) return;
  int out[4];
  phase1_row_ranges(r, b, a, out);
  blk[r] = r / b;
  pos[r] = r;  // tokens keep their original global position IDs
#pragma unroll
  for (int j = 0; j < 4; ++j) ranges[4 * r + j] = out[j];
}

// One CTA waits, through the same bounded wait the attention and decode
// kernels use, on an mbarrier that nothing arrives on: after limit_ns the
// wait gives up and records the time-out in *status; the kernel returns.
__global__ void debug_wait_probe_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    abort_flag = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
  __syncthreads();
}

// One warp per (batch, head, token) row, lanes over D. Pass 1 (lanes over
// blocks): lane s takes block s's sub-split LSEs, its max m_s and sum
// z_s = sum_k e^(l_k - m_s), hence its LSE m_s + log z_s; the tail split's
// LSE is read as written; M is the max over the splits. Pass 2 (lanes over
// D) reads every sub-split output once, the rows of several blocks issued
// before they are used (kSub = the sub-split count rounded up to 1, 2 or 4;
// a lane holds 4 rows at D = 128 and 8 at D = 64, 64 registers, so four
// CTAs fit on an SM and 4096 rows run in one wave): a block's partial is
// sum_k e^(l_k - lse_s) o_k (written to part_o), and the merged row adds
// every split with weight e^(lse_s - M)
// [pith 2WVXFXZ2, minor comment on Algorithm 2]. Fixed order, deterministic.
template <int D, int kSub>
__global__ void __launch_bounds__(256, 4) chunk_finish_kernel(
    const float* __restrict__ sub_o, const float* __restrict__ sub_lse, int nsub, int n, int tail,
    float* __restrict__ part_o, float* __restrict__ part_lse, __nv_bfloat16* __restrict__ o,
    float* __restrict__ lse, int B, int T, int Hq) {
  constexpr int kPer = D / 32;
  constexpr int kMaxSub = kSub;  // nsub <= kSub <= 4 (the cut rule makes at most 4)
  constexpr int kBlk = (D == 128 ? 4 : 8) / kSub;  // blocks whose rows are loaded together
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (warp >= B * Hq * T) return;
  const int t = warp % T;
  const size_t bh = static_cast<size_t>(warp / T);
  const int nsplit = n + tail;
  auto srow = [&](int s, int k) { return (bh * (static_cast<size_t>(n) * nsub) + s * nsub + k) * T + t; };
  auto prow = [&](int s) { return (bh * nsplit + s) * T + t; };
  auto block_lse = [&](int s) {  // lse of block s from its sub-splits
    float l[kMaxSub], m = -INFINITY;
#pragma unroll
    for (int k = 0; k < kMaxSub; ++k) {
      l[k] = (k < nsub) ? sub_lse[srow(s, k)] : -INFINITY;
      m = fmaxf(m, l[k]);
    }
    float z = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxSub; ++k) z += (l[k] == -INFINITY) ? 0.f : expf(l[k] - m);
    return (z > 0.f) ? m + logf(z) : -INFINITY;
  };
  // pass 1: block LSEs (lane s holds block s of each 32-block round), the max
  float M = tail ? part_lse[prow(n)] : -INFINITY;
  for (int s0 = 0; s0 < n; s0 += 32) {
    const int s = s0 + lane;
    const float ls = (s < n) ? block_lse(s) : -INFINITY;
    if (s < n) part_lse[prow(s)] = ls;
    M = fmaxf(M, ls);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  // pass 2: block partials, and the merged row
  float acc[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) acc[j] = 0.f;
  float zm = 0.f;
  for (int s0 = 0; s0 < n; s0 += kBlk) {
    float lsb[kBlk], w[kBlk][kMaxSub];
    float4 v[kBlk][kMaxSub][1];  // D = 128: a float4 per lane
    float2 v2[kBlk][kMaxSub];    // D = 64: a float2 per lane
#pragma unroll
    for (int i = 0; i < kBlk; ++i) {
      const int s = s0 + i;
      lsb[i] = -INFINITY;
      if (s >= n) continue;
      lsb[i] = block_lse(s);  // the same arithmetic as pass 1: the same value in every lane
#pragma unroll
      for (int k = 0; k < kMaxSub; ++k) {
        w[i][k] = 0.f;
        if (k < nsub && lsb[i] != -INFINITY) {
          const float l = sub_lse[srow(s, k)];
          w[i][k] = (l == -INFINITY) ? 0.f : expf(l - lsb[i]);
          const float* src = sub_o + srow(s, k) * D + lane * kPer;
          if constexpr (kPer == 4) v[i][k][0] = *reinterpret_cast<const float4*>(src);
          else v2[i][k] = *reinterpret_cast<const float2*>(src);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kBlk; ++i) {
      const int s = s0 + i;
      if (s >= n) continue;
      float bo[kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j) bo[j] = 0.f;
#pragma unroll
      for (int k = 0; k < kMaxSub; ++k) {
        if (w[i][k] == 0.f) continue;
        if constexpr (kPer == 4) {
          bo[0] += w[i][k] * v[i][k][0].x;
          bo[1] += w[i][k] * v[i][k][0].y;
          bo[2] += w[i][k] * v[i][k][0].z;
          bo[3] += w[i][k] * v[i][k][0].w;
        } else {
          bo[0] += w[i][k] * v2[i][k].x;
          bo[1] += w[i][k] * v2[i][k].y;
        }
      }
      float* dst = part_o + prow(s) * D + lane * kPer;
      if constexpr (kPer == 4)
        *reinterpret_cast<float4*>(dst) = make_float4(bo[0], bo[1], bo[2], bo[3]);
      else
        *reinterpret_cast<float2*>(dst) = make_float2(bo[0], bo[1]);
      if (o != nullptr && M != -INFINITY && lsb[i] != -INFINITY) {
        const float wm = expf(lsb[i] - M);
        zm += wm;
#pragma unroll
        for (int j = 0; j < kPer; ++j) acc[j] += wm * bo[j];
      }
    }
  }
  if (o == nullptr) return;
  if (tail) {
    const float ltail = part_lse[prow(n)];
    if (M != -INFINITY && ltail != -INFINITY) {
      const float wt = expf(ltail - M);
      zm += wt;
      const float* src = part_o + prow(n) * D + lane * kPer;
#pragma unroll
      for (int j = 0; j < kPer; ++j) acc[j] += wt * src[j];
    }
  }
  const float inv = (zm > 0.f) ? 1.f / zm : 0.f;
  const int b = static_cast<int>(bh / Hq), h = static_cast<int>(bh % Hq);
  __nv_bfloat16* od = o + ((static_cast<size_t>(b) * T + t) * Hq + h) * D + lane * kPer;
#pragma unroll
  for (int j = 0; j < kPer; j += 2)
    *reinterpret_cast<uint32_t*>(od + j) = pack_bf16x2(acc[j] * inv, acc[j + 1] * inv);
  if (lse != nullptr && lane == 0) lse[bh * T + t] = (zm > 0.f) ? M + logf(zm) : -INFINITY;
}

cudaError_t launch_chunk_finish(const float* sub_o, const float* sub_lse, int nsub, int n,
                                int tail, float* part_o, float* part_lse, __nv_bfloat16* o,
                                float* lse, int B, int T, int Hq, int D, cudaStream_t stream) {
  const long long rows = static_cast<long long>(B) * Hq * T;
  if (rows == 0) return cudaSuccess;
  const int threads = 256;
  const unsigned blocks = static_cast<unsigned>((rows * 32 + threads - 1) / threads);
#define STAR_CHUNK_FINISH(DD, KS)                                                              \
  chunk_finish_kernel<DD, KS><<<blocks, threads, 0, stream>>>(sub_o, sub_lse, nsub, n, tail,    \
                                                              part_o, part_lse, o, lse, B, T, Hq)
  const int ks = nsub <= 1 ? 1 : (nsub == 2 ? 2 : 4);
  if (D == 128) {
    if (ks == 1) STAR_CHUNK_FINISH(128, 1);
    else if (ks == 2) STAR_CHUNK_FINISH(128, 2);
    else STAR_CHUNK_FINISH(128, 4);
  } else {
    if (ks == 1) STAR_CHUNK_FINISH(64, 1);
    else if (ks == 2) STAR_CHUNK_FINISH(64, 2);
    else STAR_CHUNK_FINISH(64, 4);
  }
#undef STAR_CHUNK_FINISH
  return cudaGetLastError();
}

cudaError_t launch_debug_wait_probe(int* status, unsigned long long limit_ns, cudaStream_t stream) {
  debug_wait_probe_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_debug_index(int L, int b, int a, int32_t* blk, int32_t* pos, int32_t* ranges,
                               cudaStream_t stream) {
  if (L <= 0) return cudaSuccess;
  debug_index_kernel<<<ceil_div(L, 256), 256, 0, stream>>>(L, b, a, blk, pos, ranges);
  return cudaGetLastError();
}

}  // namespace star
