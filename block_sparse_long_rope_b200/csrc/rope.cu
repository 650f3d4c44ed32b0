// Rotate-half RoPE at global positions, and the copy of V into the
// head-major KV cache.
//
// The pages keep every token at its original global position ID — the anchor
// block keeps positions 0..a-1 in every augmented block [pith 2WVXFXZ2,
// "What carries the argument"], which preserves RoPE distances [pith
// 2607.20457, "What carries the argument"]. Pair (x_i, x_{i+D/2}) turns by
// p * theta^(-2i/D).
//
// Precision: the angle p * theta_i, its reduction modulo 2*pi (Cody-Waite,
// two constants) and sine/cosine are fp64. Every output is the correctly
// rounded bf16 (nearest even) of the exact rotation. The rotation first runs
// in fp32 with a bound E on its error; when y - E and y + E round to the same
// bf16 value that value is the correct rounding (Ziv's rounding test), and
// otherwise (about one element in 10^4) the element is recomputed in fp64 and
// rounded once through fp32 round-to-odd (Boldo and Melquiond, 2008: odd
// rounding to a format >= 2 bits wider, then nearest, equals direct nearest
// rounding). At p ~ 1e6 an fp32 angle would err by ~0.06 rad, and even an
// fp32 rotation with an exact angle lands one bf16 ulp off the correct value
// for a few elements in 1e5, enough to move a peaked softmax's log-sum-exp by
// ~3e-2; correct rounding makes the cache reproducible bit for bit.
// theta_i = theta^(-2i/D) comes from the host in fp64.
//
// One launch handles up to three jobs (Q, K, V of one call): blockIdx.z
// selects the job. Each CTA covers kTokPerCta tokens of one job; it first
// computes the (cos, sin) table of its tokens in shared memory, then streams
// 16-byte vectors: a thread rotates chunk c of the first half together with
// chunk c of the second half of one head.
#include <cmath>

#include "star_common.cuh"
#include "star_kernels.cuh"

namespace star {

namespace {
// fp64 -> fp32 with round-to-odd: truncate, then force the last bit to 1 if
// anything was cut off.
__device__ __forceinline__ float f32_round_odd(double x) {
  float f = __double2float_rz(x);
  if (static_cast<double>(f) != x) f = __uint_as_float(__float_as_uint(f) | 1u);
  return f;
}
constexpr int kRopeThreads = 256;
constexpr int kTokPerCta = 8;
constexpr double kTwoPiHi = 6.283185307179586;         // nearest double to 2*pi
constexpr double kTwoPiLo = 2.4492935982947064e-16;    // 2*pi - kTwoPiHi
constexpr double kInvTwoPi = 0.15915494309189535;
}  // namespace

__global__ void __launch_bounds__(kRopeThreads) rope_kernel(const __grid_constant__ RopeParams p) {
  const RopeJob& job = p.job[blockIdx.z];
  const int D = p.D, half = D / 2, cpr = half / 8;  // 16-byte chunks per half row
  const int tok0 = blockIdx.x * kTokPerCta;
  const int b = blockIdx.y;
  const int ntok = imin(kTokPerCta, p.S - tok0);
  if (ntok <= 0) return;

  __shared__ double s_cos[kTokPerCta][64];
  __shared__ double s_sin[kTokPerCta][64];
  __shared__ float f_cos[kTokPerCta][64];
  __shared__ float f_sin[kTokPerCta][64];
  if (job.rotate) {
    for (int e = threadIdx.x; e < ntok * half; e += blockDim.x) {
      int t = e / half, i = e % half;
      int s = tok0 + t;
      long long pos = p.pos ? static_cast<long long>(p.pos[s]) : p.pos0 + s;
      double ang = static_cast<double>(pos) * p.inv_freq[i];
      double k = rint(ang * kInvTwoPi);
      double r = fma(-k, kTwoPiHi, ang);
      r = fma(-k, kTwoPiLo, r);
      double sn, cs;
      sincos(r, &sn, &cs);
      s_cos[t][i] = cs;
      s_sin[t][i] = sn;
      f_cos[t][i] = static_cast<float>(cs);
      f_sin[t][i] = static_cast<float>(sn);
    }
    __syncthreads();
  }

  const int units = ntok * job.H * cpr;  // (token, head, chunk) triples
  for (int u = threadIdx.x; u < units; u += blockDim.x) {
    int c = u % cpr;
    int h = (u / cpr) % job.H;
    int t = u / (cpr * job.H);
    int s = tok0 + t;
    const __nv_bfloat16* xr = job.x + b * job.xs[0] + s * job.xs[1] + h * job.xs[2];
    __nv_bfloat16* yr = job.y + b * job.ys[0] + s * job.ys[1] + h * job.ys[2];
    uint4 lo = *reinterpret_cast<const uint4*>(xr + 8 * c);
    uint4 hi = *reinterpret_cast<const uint4*>(xr + half + 8 * c);
    if (job.rotate) {
      const uint32_t* pl = reinterpret_cast<const uint32_t*>(&lo);
      const uint32_t* ph = reinterpret_cast<const uint32_t*>(&hi);
      uint32_t ol[4], oh[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int i0 = 8 * c + 2 * w;
        const float a0 = bf16_lo(pl[w]), a1 = bf16_hi(pl[w]);
        const float b0 = bf16_lo(ph[w]), b1 = bf16_hi(ph[w]);
        const float c0 = f_cos[t][i0], c1 = f_cos[t][i0 + 1];
        const float s0 = f_sin[t][i0], s1 = f_sin[t][i0 + 1];
        // |fp32 result - exact| <= 2^-22 (|a| + |b|): one rounding each for
        // cos/sin (2^-25 relative), the product and the fused multiply-add
        const float e0 = 2.3841858e-07f * (fabsf(a0) + fabsf(b0));
        const float e1 = 2.3841858e-07f * (fabsf(a1) + fabsf(b1));
        float y[4] = {fmaf(a0, c0, -(b0 * s0)), fmaf(a1, c1, -(b1 * s1)),
                      fmaf(b0, c0, a0 * s0), fmaf(b1, c1, a1 * s1)};
        const float err[4] = {e0, e1, e0, e1};
        uint32_t out[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t lohi = pack_bf16x2(y[m] - err[m], y[m] + err[m]);
          if ((lohi & 0xFFFFu) == (lohi >> 16)) {
            out[m] = lohi & 0xFFFFu;
          } else {  // within E of a rounding boundary: decide in fp64
            const int ii = i0 + (m & 1);
            const double ad = (m & 1) ? a1 : a0, bd = (m & 1) ? b1 : b0;
            const double cd = s_cos[t][ii], sd = s_sin[t][ii];
            const double yd = (m < 2) ? ad * cd - bd * sd : bd * cd + ad * sd;
            out[m] = pack_bf16x2(f32_round_odd(yd), 0.f) & 0xFFFFu;
          }
        }
        ol[w] = out[0] | (out[1] << 16);
        oh[w] = out[2] | (out[3] << 16);
      }
      lo = make_uint4(ol[0], ol[1], ol[2], ol[3]);
      hi = make_uint4(oh[0], oh[1], oh[2], oh[3]);
    }
    *reinterpret_cast<uint4*>(yr + 8 * c) = lo;
    *reinterpret_cast<uint4*>(yr + half + 8 * c) = hi;
  }
}

void rope_set_freq(RopeParams& p, int D, double theta) {
  for (int i = 0; i < 64; ++i)
    p.inv_freq[i] = (i < D / 2) ? std::pow(theta, -2.0 * static_cast<double>(i) / static_cast<double>(D)) : 0.0;
}

cudaError_t launch_rope(const RopeParams& p, int njobs, cudaStream_t stream) {
  if (njobs <= 0 || p.S <= 0 || p.B <= 0) return cudaSuccess;
  dim3 grid(ceil_div(p.S, kTokPerCta), p.B, njobs);
  rope_kernel<<<grid, kRopeThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace star
