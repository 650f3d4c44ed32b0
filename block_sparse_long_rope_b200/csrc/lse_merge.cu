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

// One warp per (batch, head, token) row, lanes over D. Pass 1 reads the
// sub-split LSEs: each block's own max m_s and sum z_s = sum_k e^(l_k - m_s)
// give its LSE m_s + log z_s; the tail split's LSE is read as written. Pass 2
// reads every sub-split output once: a block's partial is
// sum_k e^(l_k - m_s) o_k / z_s (written to part_o), and the merged row adds
// every split with weight e^(lse_s - M), M the max over the splits
// [pith 2WVXFXZ2, minor comment on Algorithm 2]. Fixed order, deterministic.
template <int D>
__global__ void __launch_bounds__(256) chunk_finish_kernel(
    const float* __restrict__ sub_o, const float* __restrict__ sub_lse, int nsub, int n, int tail,
    float* __restrict__ part_o, float* __restrict__ part_lse, __nv_bfloat16* __restrict__ o,
    float* __restrict__ lse, int B, int T, int Hq) {
  constexpr int kPer = D / 32;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (warp >= B * Hq * T) return;
  const int t = warp % T;
  const size_t bh = static_cast<size_t>(warp / T);
  const int nsplit = n + tail;
  auto srow = [&](int s, int k) { return (bh * (static_cast<size_t>(n) * nsub) + s * nsub + k) * T + t; };
  auto prow = [&](int s) { return (bh * nsplit + s) * T + t; };
  // a block's LSE from its sub-splits (every lane computes the same value)
  auto block_lse = [&](int s) {
    float m = -INFINITY;
    for (int k = 0; k < nsub; ++k) m = fmaxf(m, sub_lse[srow(s, k)]);
    float z = 0.f;
    if (m != -INFINITY)
      for (int k = 0; k < nsub; ++k) {
        const float l = sub_lse[srow(s, k)];
        z += (l == -INFINITY) ? 0.f : expf(l - m);
      }
    return (z > 0.f) ? m + logf(z) : -INFINITY;
  };
  // pass 1: the max over the splits
  float M = -INFINITY;
  for (int s = 0; s < n; ++s) M = fmaxf(M, block_lse(s));
  const float ltail = tail ? part_lse[prow(n)] : -INFINITY;
  M = fmaxf(M, ltail);
  // pass 2: block partials, and the merged row
  float acc[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) acc[j] = 0.f;
  float zm = 0.f;
  for (int s = 0; s < n; ++s) {
    const float ls = block_lse(s);
    if (lane == 0) part_lse[prow(s)] = ls;
    float bo[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) bo[j] = 0.f;
    if (ls != -INFINITY) {
      for (int k = 0; k < nsub; ++k) {
        const float l = sub_lse[srow(s, k)];
        const float w = (l == -INFINITY) ? 0.f : expf(l - ls);  // already normalised by z_s
        const float* src = sub_o + srow(s, k) * D + lane * kPer;
        if constexpr (kPer == 4) {
          const float4 v = *reinterpret_cast<const float4*>(src);
          bo[0] += w * v.x;
          bo[1] += w * v.y;
          bo[2] += w * v.z;
          bo[3] += w * v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2*>(src);
          bo[0] += w * v.x;
          bo[1] += w * v.y;
        }
      }
    }
    float* dst = part_o + prow(s) * D + lane * kPer;
    if constexpr (kPer == 4)
      *reinterpret_cast<float4*>(dst) = make_float4(bo[0], bo[1], bo[2], bo[3]);
    else
      *reinterpret_cast<float2*>(dst) = make_float2(bo[0], bo[1]);
    if (o != nullptr && M != -INFINITY && ls != -INFINITY) {
      const float w = expf(ls - M);
      zm += w;
#pragma unroll
      for (int j = 0; j < kPer; ++j) acc[j] += w * bo[j];
    }
  }
  if (o == nullptr) return;
  if (tail && M != -INFINITY && ltail != -INFINITY) {
    const float w = expf(ltail - M);
    zm += w;
    const float* src = part_o + prow(n) * D + lane * kPer;
#pragma unroll
    for (int j = 0; j < kPer; ++j) acc[j] += w * src[j];
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
  if (D == 128)
    chunk_finish_kernel<128><<<blocks, threads, 0, stream>>>(sub_o, sub_lse, nsub, n, tail, part_o,
                                                             part_lse, o, lse, B, T, Hq);
  else
    chunk_finish_kernel<64><<<blocks, threads, 0, stream>>>(sub_o, sub_lse, nsub, n, tail, part_o,
                                                            part_lse, o, lse, B, T, Hq);
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
