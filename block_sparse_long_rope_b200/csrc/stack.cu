// The row-wise layers around Star attention in a decoder stack: RMSNorm and
// the Q/K/V/O projections (with the residual add fused into the O
// projection). Star Attention keeps the model unchanged — only attention is
// replaced [pith 2WVXFXZ2, the paper's abstract: training-free, compatible
// with most Transformer LLMs] — and every layer encodes its own anchor, so in
// a stack the anchor's hidden state at layer l is block 1's (the anchor is a
// causal prefix of every augmented block).
//
// RMSNorm: one CTA per row, fp32 sum of squares, y = x * rsqrt(mean(x^2) +
// eps) * gamma rounded to bf16. HBM-bound.
// Projections: the library's tcgen05 GEMM (gemm_sm100.cu), y[M, N] (+)=
// x[M, K] * w[N, K]^T in bf16 with fp32 accumulation; the residual add rounds
// the bf16 projection plus y once more. star_linear_rope adds the RoPE and
// KV-cache epilogues, so a layer's Q and K leave the projection already
// rotated and K/V land in the cache without a separate pass.
#include <cmath>
#include <cstdio>

#include <cstdarg>
#include <cstring>

#include "star.h"
#include "star_common.cuh"
#include "star_kernels.cuh"

namespace star {

namespace {

constexpr int kNormThreads = 256;

__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(const __nv_bfloat16* __restrict__ x,
                                                                const __nv_bfloat16* __restrict__ gamma,
                                                                __nv_bfloat16* __restrict__ y,
                                                                int dm, float eps) {
  __shared__ float red[kNormThreads / 32];
  const size_t row = blockIdx.x;
  const __nv_bfloat16* xr = x + row * dm;
  __nv_bfloat16* yr = y + row * dm;
  const int nvec = dm / 8;  // 16-byte vectors
  float ss = 0.f;
  for (int i = threadIdx.x; i < nvec; i += kNormThreads) {
    const uint4 u = reinterpret_cast<const uint4*>(xr)[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = bf16_lo(w[j]), b = bf16_hi(w[j]);
      ss = fmaf(a, a, ss);
      ss = fmaf(b, b, ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int k = 0; k < kNormThreads / 32; ++k) tot += red[k];
  const float r = rsqrtf(tot / static_cast<float>(dm) + eps);
  for (int i = threadIdx.x; i < nvec; i += kNormThreads) {
    const uint4 u = reinterpret_cast<const uint4*>(xr)[i];
    const uint4 g = reinterpret_cast<const uint4*>(gamma)[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      out[j] = pack_bf16x2(bf16_lo(w[j]) * r * bf16_lo(gw[j]), bf16_hi(w[j]) * r * bf16_hi(gw[j]));
    reinterpret_cast<uint4*>(yr)[i] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace

cudaError_t launch_rmsnorm(const __nv_bfloat16* x, const __nv_bfloat16* gamma, __nv_bfloat16* y,
                           int rows, int dm, float eps, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  rmsnorm_kernel<<<rows, kNormThreads, 0, stream>>>(x, gamma, y, dm, eps);
  return cudaGetLastError();
}

}  // namespace star

namespace {

star_status stack_fail(star_status st, const char* fmt, ...) {
  char buf[320];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  star::set_last_error(buf);
  return st;
}

bool misaligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; }

// Shared body of star_linear / star_linear_rope: checks, TMA maps, launch.
star_status run_gemm(const void* x, const void* w, void* y, int M, int N, int K, int accumulate,
                     int head_dim, int rotate, int seq_len, long long pos0, double theta,
                     int cache_rows, void* workspace, size_t workspace_bytes, void* cuda_stream,
                     void* y2 = nullptr, int n_split = 0) {
  if (M < 1 || N < 1 || K < 1 || N % 8 || K % 8)
    return stack_fail(STAR_ERR_INVALID_ARG, "bad shape M=%d N=%d K=%d (N, K multiples of 8)", M, N, K);
  if (!x || !w || !y || misaligned(x, 16) || misaligned(w, 16) || misaligned(y, 16))
    return stack_fail(STAR_ERR_INVALID_ARG, "x, w and y must be non-NULL and 16-byte aligned");
  const size_t need = star_linear_rope_workspace_bytes(seq_len, head_dim, rotate);
  if (!workspace || workspace_bytes < need || misaligned(workspace, 256))
    return stack_fail(STAR_ERR_INVALID_ARG,
                      "workspace must be 256-byte aligned with >= %zu bytes (status word%s)", need,
                      rotate ? " and cos/sin table" : "");
  if ((long long)M * N > (1ll << 46) || (long long)M * K > (1ll << 46) || (long long)N * K > (1ll << 46))
    return stack_fail(STAR_ERR_INVALID_ARG, "problem too large");
  const int sms = star::device_sms();
  if (sms <= 0) return STAR_ERR_UNSUPPORTED;  // message set by the device check
  star::GemmParams p;
  memset(&p, 0, sizeof p);
  if (!star::encode_tmap_2d(&p.tmA, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64, 128) ||
      !star::encode_tmap_2d(&p.tmB, w, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, 64, 256))
    return stack_fail(STAR_ERR_CUDA, "cuTensorMapEncodeTiled failed for the GEMM operands");
  p.M = M;
  p.N = N;
  p.K = K;
  p.m_tiles = (M + 127) / 128;
  p.n_tiles = (N + 255) / 256;
  p.k_blocks = (K + 63) / 64;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.accumulate = accumulate;
  p.rd = rotate ? head_dim : 0;
  p.hd = head_dim;
  p.seq_len = seq_len;
  p.cache_rows = cache_rows;
  p.pos0 = pos0;
  p.n_split = y2 ? n_split : N;
  p.y2 = static_cast<__nv_bfloat16*>(y2 ? y2 : y);
  p.status = static_cast<int*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e;
  if (rotate) {
    star::rope_fill_freq(p.inv_freq, head_dim, theta);
    float2* tab = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + star::kStatusBytes);
    e = star::launch_rope_table(tab, seq_len, head_dim / 2, pos0, p.inv_freq, st);
    if (e != cudaSuccess) return stack_fail(STAR_ERR_CUDA, "rope table launch: %s", cudaGetErrorString(e));
    p.rope_tab = tab;
  }
  e = star::launch_gemm(p, sms, st);
  if (e != cudaSuccess) return stack_fail(STAR_ERR_CUDA, "gemm launch: %s", cudaGetErrorString(e));
  star::set_last_error("");
  return STAR_OK;
}

}  // namespace

extern "C" {

star_status star_rmsnorm(const void* x, const void* gamma, void* y, int rows, int dm, float eps,
                         void* cuda_stream) {
  char buf[256];
  if (rows < 0 || dm < 8 || dm % 8 != 0 || !(eps >= 0.f)) {
    snprintf(buf, sizeof buf, "bad shape rows=%d dm=%d (a multiple of 8) eps=%g", rows, dm, eps);
    star::set_last_error(buf);
    return STAR_ERR_INVALID_ARG;
  }
  if (!x || !gamma || !y || (reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(gamma) |
                             reinterpret_cast<uintptr_t>(y)) & 15u) {
    star::set_last_error("x, gamma and y must be non-NULL and 16-byte aligned");
    return STAR_ERR_INVALID_ARG;
  }
  cudaError_t e = star::launch_rmsnorm(static_cast<const __nv_bfloat16*>(x),
                                       static_cast<const __nv_bfloat16*>(gamma),
                                       static_cast<__nv_bfloat16*>(y), rows, dm, eps,
                                       static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) {
    snprintf(buf, sizeof buf, "rmsnorm launch: %s", cudaGetErrorString(e));
    star::set_last_error(buf);
    return STAR_ERR_CUDA;
  }
  star::set_last_error("");
  return STAR_OK;
}

size_t star_linear_rope_workspace_bytes(int seq_len, int head_dim, int rotate) {
  if (!rotate || seq_len < 1 || head_dim < 2) return star::kStatusBytes;
  const size_t tab = (size_t)seq_len * (head_dim / 2) * 8;
  return star::kStatusBytes + (tab + 255) / 256 * 256;
}

star_status star_linear(const void* x, const void* w, void* y, int M, int N, int K, int accumulate,
                        void* workspace, size_t workspace_bytes, void* cuda_stream) {
  if (accumulate != 0 && accumulate != 1)
    return stack_fail(STAR_ERR_INVALID_ARG, "accumulate must be 0 or 1 (got %d)", accumulate);
  return run_gemm(x, w, y, M, N, K, accumulate, 64, 0, M, 0, 1.0, 0, workspace, workspace_bytes,
                  cuda_stream);
}

star_status star_linear_rope(const void* x, const void* w, void* y, int M, int N, int K,
                             int head_dim, int rotate, int seq_len, int64_t pos0, double theta,
                             int cache_rows, void* workspace, size_t workspace_bytes,
                             void* cuda_stream) {
  if (head_dim != 64 && head_dim != 128)
    return stack_fail(STAR_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", head_dim);
  if (rotate != 0 && rotate != 1)
    return stack_fail(STAR_ERR_INVALID_ARG, "rotate must be 0 or 1 (got %d)", rotate);
  if (N % head_dim) return stack_fail(STAR_ERR_INVALID_ARG, "N (%d) must be whole heads of %d", N, head_dim);
  if (seq_len < 1 || M % seq_len)
    return stack_fail(STAR_ERR_INVALID_ARG, "M (%d) must be a multiple of seq_len (%d)", M, seq_len);
  if (cache_rows != 0 && cache_rows < seq_len)
    return stack_fail(STAR_ERR_INVALID_ARG, "cache_rows (%d) must be 0 or >= seq_len (%d)",
                      cache_rows, seq_len);
  if (!rotate && cache_rows == 0)
    return stack_fail(STAR_ERR_INVALID_ARG, "neither rotation nor a cache layout: use star_linear");
  if (rotate && (pos0 < 0 || !(theta > 0.0)))
    return stack_fail(STAR_ERR_INVALID_ARG, "pos0 must be >= 0 and theta > 0");
  return run_gemm(x, w, y, M, N, K, 0, head_dim, rotate, seq_len, pos0, theta, cache_rows,
                  workspace, workspace_bytes, cuda_stream);
}

star_status star_linear_kv_cache(const void* x, const void* w_kv, void* k_cache, void* v_cache,
                                 int M, int N, int K, int head_dim, int seq_len, int64_t pos0,
                                 double theta, int cache_rows, void* workspace,
                                 size_t workspace_bytes, void* cuda_stream) {
  if (head_dim != 64 && head_dim != 128)
    return stack_fail(STAR_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", head_dim);
  if (N < 1 || N % head_dim)
    return stack_fail(STAR_ERR_INVALID_ARG, "N (%d) must be whole heads of %d", N, head_dim);
  if (seq_len < 1 || M % seq_len)
    return stack_fail(STAR_ERR_INVALID_ARG, "M (%d) must be a multiple of seq_len (%d)", M, seq_len);
  if (cache_rows < seq_len)
    return stack_fail(STAR_ERR_INVALID_ARG, "cache_rows (%d) must be >= seq_len (%d)", cache_rows,
                      seq_len);
  if (pos0 < 0 || !(theta > 0.0))
    return stack_fail(STAR_ERR_INVALID_ARG, "pos0 must be >= 0 and theta > 0");
  if (!v_cache || misaligned(v_cache, 16))
    return stack_fail(STAR_ERR_INVALID_ARG, "v_cache must be non-NULL and 16-byte aligned");
  if ((long long)N * 2 > (1ll << 30)) return stack_fail(STAR_ERR_INVALID_ARG, "N too large");
  return run_gemm(x, w_kv, k_cache, M, 2 * N, K, 0, head_dim, 1, seq_len, pos0, theta,
                  cache_rows, workspace, workspace_bytes, cuda_stream, v_cache, N);
}

}  // extern "C"
