// Rotate-half RoPE arithmetic shared by every kernel that rotates Q or K, so
// that all of them produce the same bits.
//
// Pair (x_i, x_{i+D/2}) turns by the angle p * theta_i, theta_i =
// theta^(-2i/D) (from the host, fp64). The angle, its reduction modulo 2*pi
// (Cody-Waite, two constants) and sine/cosine are fp64. Each output is the
// correctly rounded bf16 (nearest even) of the exact rotation: the rotation
// first runs in fp32 with a bound E on its error; when y - E and y + E round
// to the same bf16 value that value is the correct rounding (Ziv's rounding
// test), otherwise (about one element in 10^4) the element is recomputed in
// fp64 and rounded once through fp32 round-to-odd (Boldo and Melquiond, 2008:
// odd rounding to a format >= 2 bits wider, then nearest, equals direct
// nearest rounding).
#pragma once

#include "star_common.cuh"

namespace star {

constexpr double kTwoPiHi = 6.283185307179586;       // nearest double to 2*pi
constexpr double kTwoPiLo = 2.4492935982947064e-16;  // 2*pi - kTwoPiHi
constexpr double kInvTwoPi = 0.15915494309189535;

// cos / sin of pos * inv_freq (fp64, angle reduced to [-pi, pi]).
__device__ __forceinline__ void rope_angle(long long pos, double inv_freq, double* c, double* s) {
  const double ang = static_cast<double>(pos) * inv_freq;
  const double k = rint(ang * kInvTwoPi);
  double r = fma(-k, kTwoPiHi, ang);
  r = fma(-k, kTwoPiLo, r);
  sincos(r, s, c);
}

// fp64 -> fp32 with round-to-odd: truncate, then force the last bit to 1 if
// anything was cut off.
__device__ __forceinline__ float f32_round_odd(double x) {
  float f = __double2float_rz(x);
  if (static_cast<double>(f) != x) f = __uint_as_float(__float_as_uint(f) | 1u);
  return f;
}

// Correctly rounded bf16 bits (low 16) of a*c - b*s (first == true) or
// b*c + a*s (first == false), for bf16-exact a, b. c32/s32 are the fp32
// roundings of c64/s64.
__device__ __forceinline__ uint32_t rope_rotate_bf16(float a, float b, float c32, float s32,
                                                     double c64, double s64, bool first) {
  // |fp32 result - exact| <= 2^-22 (|a| + |b|): one rounding each for cos/sin
  // (2^-25 relative), the product and the fused multiply-add
  const float e = 2.3841858e-07f * (fabsf(a) + fabsf(b));
  const float y = first ? fmaf(a, c32, -(b * s32)) : fmaf(b, c32, a * s32);
  const uint32_t lohi = pack_bf16x2(y - e, y + e);
  if ((lohi & 0xFFFFu) == (lohi >> 16)) return lohi & 0xFFFFu;
  const double ad = a, bd = b;  // within E of a rounding boundary: decide in fp64
  const double yd = first ? ad * c64 - bd * s64 : bd * c64 + ad * s64;
  return pack_bf16x2(f32_round_odd(yd), 0.f) & 0xFFFFu;
}

// Both outputs of one pair: low 16 bits the bf16 of a*c - b*s, high 16 bits
// that of b*c + a*s, each correctly rounded exactly as rope_rotate_bf16 does.
// The error bound is shared, and the fp64 cos/sin are fetched (get64(&c,
// &s)) only when a result is within the bound of a rounding boundary.
template <typename Get64>
__device__ __forceinline__ uint32_t rope_rotate_pair_bf16_with(float a, float b, float c32,
                                                               float s32, Get64 get64) {
  const float e = 2.3841858e-07f * (fabsf(a) + fabsf(b));
  const float y0 = fmaf(a, c32, -(b * s32));
  const float y1 = fmaf(b, c32, a * s32);
  const uint32_t r0 = pack_bf16x2(y0 - e, y0 + e), r1 = pack_bf16x2(y1 - e, y1 + e);
  uint32_t o0 = r0 & 0xFFFFu, o1 = r1 & 0xFFFFu;
  const bool ok0 = o0 == (r0 >> 16), ok1 = o1 == (r1 >> 16);
  if (!(ok0 && ok1)) {
    double cd, sd;
    get64(&cd, &sd);
    const double ad = a, bd = b;
    if (!ok0) o0 = pack_bf16x2(f32_round_odd(ad * cd - bd * sd), 0.f) & 0xFFFFu;
    if (!ok1) o1 = pack_bf16x2(f32_round_odd(bd * cd + ad * sd), 0.f) & 0xFFFFu;
  }
  return o0 | (o1 << 16);
}

// As above with the fp64 cos/sin read through pointers (from a table).
__device__ __forceinline__ uint32_t rope_rotate_pair_bf16(float a, float b, float c32, float s32,
                                                          const double* c64, const double* s64) {
  return rope_rotate_pair_bf16_with(a, b, c32, s32, [&](double* c, double* s) {
    *c = *c64;
    *s = *s64;
  });
}

// The rare slow path of rope_rotate_pair_bf16_at, kept out of line so that
// unrolled callers stay small: recomputes the fp64 cos/sin of pos * inv_freq
// and rounds the outputs flagged in `need` (bit 0: first, bit 1: second)
// exactly as rope_rotate_pair_bf16_with does; `fast` holds the others.
static __device__ __noinline__ uint32_t rope_pair_exact_at(float a, float b, long long pos,
                                                    double inv_freq, uint32_t fast, uint32_t need) {
  double cd, sd;
  rope_angle(pos, inv_freq, &cd, &sd);
  const double ad = a, bd = b;
  uint32_t o0 = fast & 0xFFFFu, o1 = fast >> 16;
  if (need & 1u) o0 = pack_bf16x2(f32_round_odd(ad * cd - bd * sd), 0.f) & 0xFFFFu;
  if (need & 2u) o1 = pack_bf16x2(f32_round_odd(bd * cd + ad * sd), 0.f) & 0xFFFFu;
  return o0 | (o1 << 16);
}

// As rope_rotate_pair_bf16_with, with the fp64 cos/sin of pos * inv_freq
// recomputed on the rare slow path (c32/s32 must be the fp32 roundings of
// rope_angle's results): the same bits.
__device__ __forceinline__ uint32_t rope_rotate_pair_bf16_at(float a, float b, float c32, float s32,
                                                             long long pos, double inv_freq) {
  const float e = 2.3841858e-07f * (fabsf(a) + fabsf(b));
  const float y0 = fmaf(a, c32, -(b * s32));
  const float y1 = fmaf(b, c32, a * s32);
  const uint32_t r0 = pack_bf16x2(y0 - e, y0 + e), r1 = pack_bf16x2(y1 - e, y1 + e);
  const uint32_t o0 = r0 & 0xFFFFu, o1 = r1 & 0xFFFFu;
  const uint32_t need = (o0 == (r0 >> 16) ? 0u : 1u) | (o1 == (r1 >> 16) ? 0u : 2u);
  if (need) return rope_pair_exact_at(a, b, pos, inv_freq, o0 | (o1 << 16), need);
  return o0 | (o1 << 16);
}

}  // namespace star
