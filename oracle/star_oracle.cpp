// Star Attention oracle: plain, slow, fp64 CPU restatement of the method.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
// this file; only the tests, the smoke check and the benchmark's CPU-baseline
// leg do. It shares no code, header, table or constant with the CUDA library.
//
// Every function follows the definitions on the pages about Star Attention
// (arXiv 2411.17116), cited as "page, section":
//   [pith 2WVXFXZ2, "What carries the argument"]  anchor block c1 prefixed to
//       every later block with its original position indices; each block
//       attends only inside its augmented block; the anchor's KV is dropped.
//   [pith 2WVXFXZ2, minor comment on Section 2.1]  c'_1 = c_1 (b tokens);
//       only blocks i >= 2 carry the anchor.
//   [pith 2WVXFXZ2, Referee summary / Circularity check]  phase 2: each host
//       returns a local attention output and a softmax statistic; the query
//       host re-weights them into exact global attention.
//   [pith 2WVXFXZ2, minor comment on Algorithm 2]  the update weight is
//       exp(s_h - s_global), so s is a log-domain statistic.
//   [pith 2WVXFXZ2, abstract]  query and response tokens attend to all prior
//       cached tokens.
//   [pith 2607.20457, "What carries the argument"]  original global position
//       IDs preserve RoPE distances.
// Readings where the pages are silent (softmax scale 1/sqrt(D), rotate-half
// RoPE with pairs (i, i+D/2), GQA head h -> kv head h/g, query and decode
// tokens at consecutive positions after the context, bf16 storage of the
// rotated Q/K) are the plainest ones and are listed with the design notes.
//
// Arithmetic is fp64 throughout; softmax is the two-pass form (max, then
// sum) over the explicit visible key set: no tiling, no online softmax.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <map>
#include <utility>
#include <vector>

namespace {

using i64 = int64_t;
const double kNegInf = -std::numeric_limits<double>::infinity();

// bf16 bit pattern -> exact double (bf16 is the top half of an IEEE float).
double bf16_to_double(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

// Round a double to the nearest bf16 value, ties to even, in one step (no
// intermediate float). bf16 keeps 8 significant bits and the float exponent
// range: normals down to 2^-126, subnormal spacing 2^-133, max (2-2^-7)*2^127.
double round_to_bf16(double x) {
  if (!std::isfinite(x) || x == 0.0) return x;
  int e = 0;
  std::frexp(x, &e);                    // |x| = f * 2^e with f in [0.5, 1)
  int ulp_exp = std::max(e - 8, -133);  // weight of the last kept bit
  double scaled = std::ldexp(x, -ulp_exp);
  double r = std::nearbyint(scaled);    // default mode: nearest, ties to even
  double y = std::ldexp(r, ulp_exp);
  const double bf16_max = 3.3895313892515355e38;
  if (std::fabs(y) > bf16_max) return std::copysign(INFINITY, x);
  return y;
}

// Rotate-half RoPE of one head vector at position p (fp64):
//   theta_i = theta^(-2i/D), i < D/2
//   y_i       = x_i cos(p theta_i) - x_{i+D/2} sin(p theta_i)
//   y_{i+D/2} = x_{i+D/2} cos(p theta_i) + x_i sin(p theta_i)
void rope_vec(const double* x, double* y, i64 D, double p, double theta) {
  const i64 h = D / 2;
  for (i64 i = 0; i < h; ++i) {
    double th = std::pow(theta, -2.0 * static_cast<double>(i) / static_cast<double>(D));
    double ang = p * th;
    double c = std::cos(ang), s = std::sin(ang);
    double a = x[i], b = x[i + h];
    y[i] = a * c - b * s;
    y[i + h] = b * c + a * s;
  }
}

struct Range {
  i64 lo, hi;  // half-open [lo, hi)
};

// Two-pass softmax attention of one query over the keys in `ranges`.
// key(c), val(c) return row pointers of length D. Writes o[D] (normalised)
// and lse (natural log). An empty key set gives lse = -inf and o = 0.
template <class KeyFn, class ValFn>
void attend(const double* q, i64 D, double scale, const std::vector<Range>& ranges, KeyFn key,
            ValFn val, double* o, double* lse, i64* nvis) {
  std::vector<double> s;
  std::vector<i64> idx;
  for (const Range& r : ranges)
    for (i64 c = r.lo; c < r.hi; ++c) {
      const double* k = key(c);
      double acc = 0.0;
      for (i64 d = 0; d < D; ++d) acc += q[d] * k[d];
      s.push_back(acc * scale);
      idx.push_back(c);
    }
  if (nvis) *nvis = static_cast<i64>(s.size());
  for (i64 d = 0; d < D; ++d) o[d] = 0.0;
  if (s.empty()) {
    *lse = kNegInf;
    return;
  }
  double m = *std::max_element(s.begin(), s.end());
  double z = 0.0;
  for (size_t j = 0; j < s.size(); ++j) {
    double w = std::exp(s[j] - m);
    z += w;
    const double* v = val(idx[j]);
    for (i64 d = 0; d < D; ++d) o[d] += w * v[d];
  }
  for (i64 d = 0; d < D; ++d) o[d] /= z;
  *lse = m + std::log(z);
}

// Phase-1 visible keys of context row r ([pith 2WVXFXZ2, "What carries the
// argument"] and the minor comment on Section 2.1):
//   block 0 (c'_1 = c_1):  keys [0, r]
//   block i >= 1:          anchor keys [0, a) at their original positions,
//                          then the own block, causally: [i*b, r]
std::vector<Range> phase1_visible(i64 r, i64 b, i64 a) {
  i64 blk = r / b;
  std::vector<Range> v;
  if (blk == 0) {
    v.push_back({0, r + 1});
  } else {
    if (a > 0) v.push_back({0, a});
    v.push_back({blk * b, r + 1});
  }
  return v;
}

// Roped (and optionally bf16-rounded) key rows [0, n) of one (batch, kv head).
std::vector<double> rope_rows(const uint16_t* k_bits, i64 b, i64 kvh, i64 n, i64 S, i64 H, i64 D,
                              i64 pos0, double theta, bool round_bf16) {
  std::vector<double> out(static_cast<size_t>(n * D));
#pragma omp parallel for schedule(static)
  for (i64 c = 0; c < n; ++c) {
    std::vector<double> x(D);
    const uint16_t* src = k_bits + ((b * S + c) * H + kvh) * D;
    for (i64 d = 0; d < D; ++d) x[d] = bf16_to_double(src[d]);
    double* y = out.data() + c * D;
    rope_vec(x.data(), y, D, static_cast<double>(pos0 + c), theta);
    if (round_bf16)
      for (i64 d = 0; d < D; ++d) y[d] = round_to_bf16(y[d]);
  }
  return out;
}

std::vector<double> plain_rows(const uint16_t* v_bits, i64 b, i64 kvh, i64 n, i64 S, i64 H, i64 D) {
  std::vector<double> out(static_cast<size_t>(n * D));
#pragma omp parallel for schedule(static)
  for (i64 c = 0; c < n; ++c) {
    const uint16_t* src = v_bits + ((b * S + c) * H + kvh) * D;
    for (i64 d = 0; d < D; ++d) out[c * D + d] = bf16_to_double(src[d]);
  }
  return out;
}

}  // namespace

extern "C" {

// bf16 rounding of n doubles in place (ties to even, single rounding).
void orc_round_bf16(double* x, i64 n) {
  for (i64 i = 0; i < n; ++i) x[i] = round_to_bf16(x[i]);
}

// y[B,S,H,D] = RoPE(x) with x given as bf16 bits; position of token s is
// pos[s]. Optionally rounds the result to bf16.
void orc_rope(const uint16_t* x_bits, i64 B, i64 S, i64 H, i64 D, const i64* pos, double theta,
              int round_bf16, double* y) {
#pragma omp parallel for collapse(2) schedule(static)
  for (i64 b = 0; b < B; ++b)
    for (i64 s = 0; s < S; ++s)
      for (i64 h = 0; h < H; ++h) {
        std::vector<double> x(D);
        const uint16_t* src = x_bits + ((b * S + s) * H + h) * D;
        for (i64 d = 0; d < D; ++d) x[d] = bf16_to_double(src[d]);
        double* dst = y + ((b * S + s) * H + h) * D;
        rope_vec(x.data(), dst, D, static_cast<double>(pos[s]), theta);
        if (round_bf16)
          for (i64 d = 0; d < D; ++d) dst[d] = round_to_bf16(dst[d]);
      }
}

// Visible-key count and key ranges of context row r under Phase 1.
// ranges_out[4] = {anchor_lo, anchor_hi, own_lo, own_hi}; block 0 reports an
// empty anchor range [0, 0).
void orc_phase1_ranges(i64 L, i64 block_len, i64 anchor_len, i64* blk, i64* ranges) {
  for (i64 r = 0; r < L; ++r) {
    std::vector<Range> v = phase1_visible(r, block_len, anchor_len);
    blk[r] = r / block_len;
    if (blk[r] == 0) {
      ranges[4 * r + 0] = 0;
      ranges[4 * r + 1] = 0;
      ranges[4 * r + 2] = v[0].lo;
      ranges[4 * r + 3] = v[0].hi;
    } else {
      ranges[4 * r + 0] = 0;
      ranges[4 * r + 1] = anchor_len;
      ranges[4 * r + 2] = v.back().lo;
      ranges[4 * r + 3] = v.back().hi;
    }
  }
}

// Phase 1 (anchor-block blockwise-local causal encoding) for a list of
// (batch, q head, row) queries. Inputs are the pre-RoPE bf16 tensors
// q[B,L,Hq,D], k/v[B,L,Hkv,D]; token t sits at position t (the anchor keeps
// positions 0..a-1). If round_qk, rotated Q and K are rounded to bf16 (the
// precision the rotated tensors and the KV cache are stored in).
// Outputs: o[nq, D], lse[nq] (natural log), nvis[nq] (nullable).
// q_sel != 0 means q_bits holds only the listed queries' vectors, [nq, D].
static void phase1_rows_impl(const uint16_t* q_bits, int q_sel, const uint16_t* k_bits,
                             const uint16_t* v_bits, i64 L, i64 Hq, i64 Hkv, i64 D, i64 block_len,
                             i64 anchor_len, double theta, int round_qk, i64 nq, const i64* qb,
                             const i64* qh, const i64* qr, double* o, double* lse, i64* nvis) {
  const i64 g = Hq / Hkv;
  const double scale = 1.0 / std::sqrt(static_cast<double>(D));
  // Group queries by (batch, kv head) so each group's keys are rotated once.
  std::map<std::pair<i64, i64>, std::vector<i64>> groups;
  for (i64 i = 0; i < nq; ++i) groups[{qb[i], qh[i] / g}].push_back(i);
  for (auto& kv : groups) {
    i64 b = kv.first.first, kvh = kv.first.second;
    i64 nmax = 0;
    for (i64 i : kv.second) nmax = std::max(nmax, qr[i] + 1);
    std::vector<double> K = rope_rows(k_bits, b, kvh, nmax, L, Hkv, D, 0, theta, round_qk != 0);
    std::vector<double> V = plain_rows(v_bits, b, kvh, nmax, L, Hkv, D);
    const std::vector<i64>& qs = kv.second;
#pragma omp parallel for schedule(dynamic, 1)
    for (size_t j = 0; j < qs.size(); ++j) {
      i64 i = qs[j];
      std::vector<double> x(D), q(D);
      const uint16_t* src = q_sel ? q_bits + i * D : q_bits + ((b * L + qr[i]) * Hq + qh[i]) * D;
      for (i64 d = 0; d < D; ++d) x[d] = bf16_to_double(src[d]);
      rope_vec(x.data(), q.data(), D, static_cast<double>(qr[i]), theta);
      if (round_qk)
        for (i64 d = 0; d < D; ++d) q[d] = round_to_bf16(q[d]);
      std::vector<Range> vis = phase1_visible(qr[i], block_len, anchor_len);
      attend(
          q.data(), D, scale, vis, [&](i64 c) { return K.data() + c * D; },
          [&](i64 c) { return V.data() + c * D; }, o + i * D, lse + i, nvis ? nvis + i : nullptr);
    }
  }
}

void orc_phase1_rows(const uint16_t* q_bits, const uint16_t* k_bits, const uint16_t* v_bits, i64 B,
                     i64 L, i64 Hq, i64 Hkv, i64 D, i64 block_len, i64 anchor_len, double theta,
                     int round_qk, i64 nq, const i64* qb, const i64* qh, const i64* qr, double* o,
                     double* lse, i64* nvis) {
  (void)B;
  phase1_rows_impl(q_bits, 0, k_bits, v_bits, L, Hq, Hkv, D, block_len, anchor_len, theta,
                   round_qk, nq, qb, qh, qr, o, lse, nvis);
}

// As orc_phase1_rows, with q_sel_bits[nq, D] holding only the listed queries.
void orc_phase1_rows_sel(const uint16_t* q_sel_bits, const uint16_t* k_bits,
                         const uint16_t* v_bits, i64 L, i64 Hq, i64 Hkv, i64 D, i64 block_len,
                         i64 anchor_len, double theta, int round_qk, i64 nq, const i64* qb,
                         const i64* qh, const i64* qr, double* o, double* lse, i64* nvis) {
  phase1_rows_impl(q_sel_bits, 1, k_bits, v_bits, L, Hq, Hkv, D, block_len, anchor_len, theta,
                   round_qk, nq, qb, qh, qr, o, lse, nvis);
}

// Generalised Phase 1 (gathered prefix). A prefix table of G rows: row g
// holds the key/value of context row src[g] (src[g] >= 0) or of extra row
// -1 - src[g] (xk/xv[B, NX, Hkv, D]), and its key is rotated at position
// pos[g]. Row r of block i = r / b sees
//   the prefix rows g in [bounds[2i], bounds[2i+1])   (all visible)
//   U [i*b, r]                                        (own block, causal)
// The Star anchor is the table of rows 0..a-1 at their own positions, seen
// by every block i >= 1 (pith 2WVXFXZ2, "What carries the argument"); the
// anchor ablations (atlas.scime.ai summary, measured-effects table) remove
// it, move its position IDs or replace its content; Pulsar's layout
// [sink || Sigma_0 || ... || Sigma_{i-1} || B_i] is the table sink, Sigma_0,
// Sigma_1, ... with block i seeing its first 64 + |Sigma_0| + ... +
// |Sigma_{i-1}| rows, every row at its original global position (pith
// 2607.20457, "What carries the argument"). A row listed twice counts twice.
// Key index c < L is context row c (own block), c >= L is prefix row c - L.
void orc_phase1_gather_rows(const uint16_t* q_bits, const uint16_t* k_bits,
                            const uint16_t* v_bits, i64 L, i64 Hq, i64 Hkv, i64 D, i64 block_len,
                            const i64* src, const i64* pos, i64 G, const i64* bounds,
                            const uint16_t* xk_bits, const uint16_t* xv_bits, i64 NX, double theta,
                            int round_qk, i64 nq, const i64* qb, const i64* qh, const i64* qr,
                            double* o, double* lse, i64* nvis) {
  const i64 g = Hq / Hkv;
  const double scale = 1.0 / std::sqrt(static_cast<double>(D));
  std::map<std::pair<i64, i64>, std::vector<i64>> groups;
  for (i64 i = 0; i < nq; ++i) groups[{qb[i], qh[i] / g}].push_back(i);
  for (auto& kv : groups) {
    const i64 b = kv.first.first, kvh = kv.first.second;
    i64 nmax = 0;
    for (i64 i : kv.second) nmax = std::max(nmax, qr[i] + 1);
    std::vector<double> K = rope_rows(k_bits, b, kvh, nmax, L, Hkv, D, 0, theta, round_qk != 0);
    std::vector<double> V = plain_rows(v_bits, b, kvh, nmax, L, Hkv, D);
    // the prefix table of this (batch, kv head)
    std::vector<double> PK(static_cast<size_t>(G * D)), PV(static_cast<size_t>(G * D));
    for (i64 t = 0; t < G; ++t) {
      const uint16_t* ks = src[t] >= 0 ? k_bits + ((b * L + src[t]) * Hkv + kvh) * D
                                       : xk_bits + ((b * NX + (-1 - src[t])) * Hkv + kvh) * D;
      const uint16_t* vs = src[t] >= 0 ? v_bits + ((b * L + src[t]) * Hkv + kvh) * D
                                       : xv_bits + ((b * NX + (-1 - src[t])) * Hkv + kvh) * D;
      std::vector<double> x(D);
      for (i64 d = 0; d < D; ++d) x[d] = bf16_to_double(ks[d]);
      rope_vec(x.data(), PK.data() + t * D, D, static_cast<double>(pos[t]), theta);
      if (round_qk)
        for (i64 d = 0; d < D; ++d) PK[t * D + d] = round_to_bf16(PK[t * D + d]);
      for (i64 d = 0; d < D; ++d) PV[t * D + d] = bf16_to_double(vs[d]);
    }
    auto key = [&](i64 c) { return c < L ? K.data() + c * D : PK.data() + (c - L) * D; };
    auto val = [&](i64 c) { return c < L ? V.data() + c * D : PV.data() + (c - L) * D; };
    const std::vector<i64>& qs = kv.second;
#pragma omp parallel for schedule(dynamic, 1)
    for (size_t j = 0; j < qs.size(); ++j) {
      const i64 i = qs[j], r = qr[i], blk = r / block_len;
      std::vector<double> x(D), q(D);
      const uint16_t* qsrc = q_bits + ((b * L + r) * Hq + qh[i]) * D;
      for (i64 d = 0; d < D; ++d) x[d] = bf16_to_double(qsrc[d]);
      rope_vec(x.data(), q.data(), D, static_cast<double>(r), theta);
      if (round_qk)
        for (i64 d = 0; d < D; ++d) q[d] = round_to_bf16(q[d]);
      std::vector<Range> vis;
      const i64 gs = bounds[2 * blk], ge = bounds[2 * blk + 1];
      if (ge > gs) vis.push_back({L + gs, L + ge});
      vis.push_back({blk * block_len, r + 1});
      attend(q.data(), D, scale, vis, key, val, o + i * D, lse + i, nvis ? nvis + i : nullptr);
    }
  }
}

// Phase 2 partials ([pith 2WVXFXZ2, Referee summary and Circularity check]):
// for new token t of this call (query or decode; position L + tail_len + t),
// one (normalised output, LSE) pair per split:
//   split j < n : context block j, keys [j*b, min((j+1)*b, L)), all visible
//   split n     : the tail (earlier query/decode tokens and this call's
//                 tokens), keys at positions L .. L + tail_len + t (causal)
// Inputs: q_new[B,T,Hq,D]; context k/v[B,L,Hkv,D]; tail k/v[B,Ltail,Hkv,D]
// holding tail tokens 0..Ltail-1 at positions L + j (Ltail >= tail_len + T).
// Outputs: part_o[nq, nsplit, D], part_lse[nq, nsplit] with nsplit = n + 1.
void orc_phase2_rows(const uint16_t* qn_bits, const uint16_t* kc_bits, const uint16_t* vc_bits,
                     const uint16_t* kt_bits, const uint16_t* vt_bits, i64 B, i64 L, i64 Ltail,
                     i64 T, i64 Hq, i64 Hkv, i64 D, i64 block_len, i64 tail_len, double theta,
                     int round_qk, i64 nq, const i64* qb, const i64* qh, const i64* qt,
                     double* part_o, double* part_lse) {
  const i64 g = Hq / Hkv;
  const i64 n = (L + block_len - 1) / block_len;
  const i64 nsplit = n + 1;
  const double scale = 1.0 / std::sqrt(static_cast<double>(D));
  std::map<std::pair<i64, i64>, std::vector<i64>> groups;
  for (i64 i = 0; i < nq; ++i) groups[{qb[i], qh[i] / g}].push_back(i);
  for (auto& kv : groups) {
    i64 b = kv.first.first, kvh = kv.first.second;
    std::vector<double> Kc = rope_rows(kc_bits, b, kvh, L, L, Hkv, D, 0, theta, round_qk != 0);
    std::vector<double> Vc = plain_rows(vc_bits, b, kvh, L, L, Hkv, D);
    i64 nt = tail_len + T;
    std::vector<double> Kt = rope_rows(kt_bits, b, kvh, nt, Ltail, Hkv, D, L, theta, round_qk != 0);
    std::vector<double> Vt = plain_rows(vt_bits, b, kvh, nt, Ltail, Hkv, D);
    const std::vector<i64>& qs = kv.second;
#pragma omp parallel for schedule(dynamic, 1)
    for (size_t jq = 0; jq < qs.size(); ++jq) {
      i64 i = qs[jq];
      i64 t = qt[i];
      std::vector<double> x(D), q(D);
      const uint16_t* src = qn_bits + ((b * T + t) * Hq + qh[i]) * D;
      for (i64 d = 0; d < D; ++d) x[d] = bf16_to_double(src[d]);
      rope_vec(x.data(), q.data(), D, static_cast<double>(L + tail_len + t), theta);
      if (round_qk)
        for (i64 d = 0; d < D; ++d) q[d] = round_to_bf16(q[d]);
      for (i64 j = 0; j < n; ++j) {
        std::vector<Range> vis{{j * block_len, std::min((j + 1) * block_len, L)}};
        attend(
            q.data(), D, scale, vis, [&](i64 c) { return Kc.data() + c * D; },
            [&](i64 c) { return Vc.data() + c * D; }, part_o + (i * nsplit + j) * D,
            part_lse + i * nsplit + j, nullptr);
      }
      std::vector<Range> tail{{0, tail_len + t + 1}};
      attend(
          q.data(), D, scale, tail, [&](i64 c) { return Kt.data() + c * D; },
          [&](i64 c) { return Vt.data() + c * D; }, part_o + (i * nsplit + n) * D,
          part_lse + i * nsplit + n, nullptr);
    }
  }
}

// One-shot softmax attention of new token t over every cached key (context
// [0, L) and tail [0, tail_len + t]) — the global attention the merge must
// reproduce exactly ([pith 2WVXFXZ2, assumptions: online softmax aggregation
// yields the exact global softmax]). Outputs o[nq, D], lse[nq].
void orc_global_rows(const uint16_t* qn_bits, const uint16_t* kc_bits, const uint16_t* vc_bits,
                     const uint16_t* kt_bits, const uint16_t* vt_bits, i64 B, i64 L, i64 Ltail,
                     i64 T, i64 Hq, i64 Hkv, i64 D, i64 tail_len, double theta, int round_qk,
                     i64 nq, const i64* qb, const i64* qh, const i64* qt, double* o, double* lse) {
  const i64 g = Hq / Hkv;
  const double scale = 1.0 / std::sqrt(static_cast<double>(D));
  std::map<std::pair<i64, i64>, std::vector<i64>> groups;
  for (i64 i = 0; i < nq; ++i) groups[{qb[i], qh[i] / g}].push_back(i);
  for (auto& kv : groups) {
    i64 b = kv.first.first, kvh = kv.first.second;
    i64 nt = tail_len + T;
    // Concatenate context and tail keys into one sequence of positions 0..L+nt-1.
    std::vector<double> Kc = rope_rows(kc_bits, b, kvh, L, L, Hkv, D, 0, theta, round_qk != 0);
    std::vector<double> Vc = plain_rows(vc_bits, b, kvh, L, L, Hkv, D);
    std::vector<double> Kt = rope_rows(kt_bits, b, kvh, nt, Ltail, Hkv, D, L, theta, round_qk != 0);
    std::vector<double> Vt = plain_rows(vt_bits, b, kvh, nt, Ltail, Hkv, D);
    auto key = [&](i64 c) { return c < L ? Kc.data() + c * D : Kt.data() + (c - L) * D; };
    auto val = [&](i64 c) { return c < L ? Vc.data() + c * D : Vt.data() + (c - L) * D; };
    const std::vector<i64>& qs = kv.second;
#pragma omp parallel for schedule(dynamic, 1)
    for (size_t jq = 0; jq < qs.size(); ++jq) {
      i64 i = qs[jq];
      i64 t = qt[i];
      std::vector<double> x(D), q(D);
      const uint16_t* src = qn_bits + ((b * T + t) * Hq + qh[i]) * D;
      for (i64 d = 0; d < D; ++d) x[d] = bf16_to_double(src[d]);
      rope_vec(x.data(), q.data(), D, static_cast<double>(L + tail_len + t), theta);
      if (round_qk)
        for (i64 d = 0; d < D; ++d) q[d] = round_to_bf16(q[d]);
      std::vector<Range> all{{0, L + tail_len + t + 1}};
      attend(q.data(), D, scale, all, key, val, o + i * D, lse + i, nullptr);
    }
  }
}

// LSE merge ([pith 2WVXFXZ2, minor comment on Algorithm 2, corrected form]):
//   m = max_h lse_h;  w_h = exp(lse_h - m);  lse = m + log(sum_h w_h)
//   o = sum_h w_h o_h / sum_h w_h
// Splits with lse = -inf get weight 0. part_o[R, nsplit, D], part_lse[R, nsplit].
void orc_lse_merge(const double* part_o, const double* part_lse, i64 R, i64 nsplit, i64 D,
                   double* o, double* lse) {
  for (i64 r = 0; r < R; ++r) {
    double m = kNegInf;
    for (i64 h = 0; h < nsplit; ++h) m = std::max(m, part_lse[r * nsplit + h]);
    for (i64 d = 0; d < D; ++d) o[r * D + d] = 0.0;
    if (m == kNegInf) {
      lse[r] = kNegInf;
      continue;
    }
    double z = 0.0;
    for (i64 h = 0; h < nsplit; ++h) {
      double l = part_lse[r * nsplit + h];
      if (l == kNegInf) continue;
      double w = std::exp(l - m);
      z += w;
      for (i64 d = 0; d < D; ++d) o[r * D + d] += w * part_o[(r * nsplit + h) * D + d];
    }
    for (i64 d = 0; d < D; ++d) o[r * D + d] /= z;
    lse[r] = m + std::log(z);
  }
}

}  // extern "C"
