// Rotate-half RoPE at global positions, and the copy of V into the
// head-major KV cache.
//
// The pages keep every token at its original global position ID — the anchor
// block keeps positions 0..a-1 in every augmented block [pith 2WVXFXZ2,
// "What carries the argument"], which preserves RoPE distances [pith
// 2607.20457, "What carries the argument"]. Pair (x_i, x_{i+D/2}) turns by
// p * theta^(-2i/D).
//
// Precision: see rope_math.cuh (fp64 angles and sine/cosine; every output
// is the correctly rounded bf16 of the exact rotation). At p ~ 1e6 an fp32
// angle would err by ~0.06 rad, and even an fp32 rotation with an exact
// angle lands one bf16 ulp off the correct value for a few elements in 1e5,
// enough to move a peaked softmax's log-sum-exp by ~3e-2; correct rounding
// makes the cache reproducible bit for bit.
//
// In gather mode the output token s takes its input row from an index
// table (a context row or a given row) and is rotated at pos[s]: this builds
// the gathered prefix table of the generalised Phase 1 (Pulsar's sink and
// summaries keep their original global positions [pith 2607.20457, "What
// carries the argument"]).
//
// One launch handles up to three jobs (Q, K, V of one call): blockIdx.z
// selects the job. Each CTA covers p.tpc tokens of one job (8 for long
// sequences, fewer for a handful of new tokens so that the grid still fills
// the GPU); it first computes the (cos, sin) table of its tokens in shared
// memory, then streams 16-byte vectors: a thread rotates chunk c of the first
// half together with chunk c of the second half of one head.
#include <cmath>

#include "rope_math.cuh"
#include "star_common.cuh"
#include "star_kernels.cuh"

namespace star {

namespace {
constexpr int kRopeThreads = 256;
}  // namespace

template <int D>
__global__ void __launch_bounds__(kRopeThreads) rope_kernel(const __grid_constant__ RopeParams p) {
  constexpr int kHalf = D / 2, kCpr = kHalf / 8;  // 16-byte chunks per half row
  const RopeJob& job = p.job[blockIdx.z];
  const int tok0 = blockIdx.x * p.tpc;
  const int b = blockIdx.y;
  const int ntok = imin(p.tpc, p.S - tok0);
  if (ntok <= 0) return;

  __shared__ double s_cos[kRopeMaxTok][64];
  __shared__ double s_sin[kRopeMaxTok][64];
  __shared__ float f_cos[kRopeMaxTok][64];
  __shared__ float f_sin[kRopeMaxTok][64];
  __shared__ int s_row[kRopeMaxTok];  // gather mode: source row, >= 0 in x, < 0 in x2
  __shared__ int s_ok[kRopeMaxTok];
  if (p.src) {
    if (threadIdx.x < ntok) {
      const int r = p.src[tok0 + threadIdx.x];
      const bool ok = (r >= 0 && r < p.nsrc) || (r < 0 && r >= -p.nx);
      s_row[threadIdx.x] = r;
      s_ok[threadIdx.x] = ok;
      if (!ok && blockIdx.z == 0) atomicOr(p.status, kDevBounds);
    }
    __syncthreads();
  }
  if (job.rotate) {
    for (int e = threadIdx.x; e < ntok * kHalf; e += kRopeThreads) {
      const int t = e / kHalf, i = e % kHalf;
      const int s = tok0 + t;
      const long long pos = p.pos ? static_cast<long long>(p.pos[s]) : p.pos0 + s;
      double sn, cs;
      rope_angle(pos, p.inv_freq[i], &cs, &sn);
      s_cos[t][i] = cs;
      s_sin[t][i] = sn;
      f_cos[t][i] = static_cast<float>(cs);
      f_sin[t][i] = static_cast<float>(sn);
    }
    __syncthreads();
  }

  // units (token, head, chunk): the token by one multiply-high with a magic
  // number (exact: u * per_tok < 2^32), head and chunk by constant shifts
  const unsigned per_tok = static_cast<unsigned>(job.H) * kCpr;
  const unsigned units = static_cast<unsigned>(ntok) * per_tok;
  const unsigned magic = 0xFFFFFFFFu / per_tok + 1u;
  for (unsigned u = threadIdx.x; u < units; u += kRopeThreads) {
    const int t = static_cast<int>(__umulhi(u, magic));
    const unsigned rem = u - static_cast<unsigned>(t) * per_tok;
    const int h = static_cast<int>(rem / kCpr), c = static_cast<int>(rem % kCpr);
    const int s = tok0 + t;
    __nv_bfloat16* yr = job.y + b * job.ys[0] + s * job.ys[1] + h * job.ys[2];
    const __nv_bfloat16* xr;
    if (!p.src) {
      xr = job.x + b * job.xs[0] + s * job.xs[1] + h * job.xs[2];
    } else if (!s_ok[t]) {
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(yr + 8 * c) = z;
      *reinterpret_cast<uint4*>(yr + kHalf + 8 * c) = z;
      continue;
    } else {
      const int r = s_row[t];
      xr = (r >= 0) ? job.x + b * job.xs[0] + r * job.xs[1] + h * job.xs[2]
                    : job.x2 + b * job.x2s[0] + (-1 - r) * job.x2s[1] + h * job.x2s[2];
    }
    uint4 lo = *reinterpret_cast<const uint4*>(xr + 8 * c);
    uint4 hi = *reinterpret_cast<const uint4*>(xr + kHalf + 8 * c);
    if (job.rotate) {
      const uint32_t* pl = reinterpret_cast<const uint32_t*>(&lo);
      const uint32_t* ph = reinterpret_cast<const uint32_t*>(&hi);
      uint32_t ol[4], oh[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int i0 = 8 * c + 2 * w;
        const uint32_t p0 = rope_rotate_pair_bf16(bf16_lo(pl[w]), bf16_lo(ph[w]), f_cos[t][i0],
                                                  f_sin[t][i0], &s_cos[t][i0], &s_sin[t][i0]);
        const uint32_t p1 = rope_rotate_pair_bf16(bf16_hi(pl[w]), bf16_hi(ph[w]), f_cos[t][i0 + 1],
                                                  f_sin[t][i0 + 1], &s_cos[t][i0 + 1],
                                                  &s_sin[t][i0 + 1]);
        ol[w] = __byte_perm(p0, p1, 0x5410);  // first outputs of both pairs
        oh[w] = __byte_perm(p0, p1, 0x7632);  // second outputs
      }
      lo = make_uint4(ol[0], ol[1], ol[2], ol[3]);
      hi = make_uint4(oh[0], oh[1], oh[2], oh[3]);
    }
    *reinterpret_cast<uint4*>(yr + 8 * c) = lo;
    *reinterpret_cast<uint4*>(yr + kHalf + 8 * c) = hi;
  }
}

void rope_fill_freq(double* out, int D, double theta) {
  for (int i = 0; i < 64; ++i)
    out[i] = (i < D / 2) ? std::pow(theta, -2.0 * static_cast<double>(i) / static_cast<double>(D)) : 0.0;
}

cudaError_t launch_rope(const RopeParams& p_in, int njobs, cudaStream_t stream) {
  if (njobs <= 0 || p_in.S <= 0 || p_in.B <= 0) return cudaSuccess;
  RopeParams p = p_in;
  if (p.tpc <= 0 || p.tpc > kRopeMaxTok) {
    // 8 tokens per CTA amortise the cos/sin table; a short call (a query
    // chunk) takes fewer so that its grid still covers two waves of CTAs
    p.tpc = kRopeMaxTok;
    while (p.tpc > 1 && (long long)ceil_div(p.S, p.tpc) * p.B * njobs < 2 * 148) p.tpc /= 2;
  }
  dim3 grid(ceil_div(p.S, p.tpc), p.B, njobs);
  if (p.D == 128)
    rope_kernel<128><<<grid, kRopeThreads, 0, stream>>>(p);
  else
    rope_kernel<64><<<grid, kRopeThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace star
