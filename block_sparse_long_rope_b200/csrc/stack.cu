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
// Projections: plain GEMMs, y[M, N] (+)= x[M, K] * w[N, K]^T in bf16 with fp32
// accumulation, through cuBLASLt; the residual is its beta = 1 term. Split-K
// algorithms are limited to fp32 reductions, so the only bf16 rounding is the
// final one.
#include <cublasLt.h>

#include <cstdio>
#include <map>
#include <mutex>
#include <tuple>

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

// ---- cuBLASLt --------------------------------------------------------------
std::mutex g_lt_mu;
cublasLtHandle_t g_lt = nullptr;
using AlgoKey = std::tuple<int, int, int, int, int, size_t>;  // device, M, N, K, beta, workspace
std::map<AlgoKey, cublasLtMatmulAlgo_t> g_algos;

struct LtDescs {
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t a = nullptr, b = nullptr, c = nullptr;
  ~LtDescs() {
    if (c) cublasLtMatrixLayoutDestroy(c);
    if (b) cublasLtMatrixLayoutDestroy(b);
    if (a) cublasLtMatrixLayoutDestroy(a);
    if (op) cublasLtMatmulDescDestroy(op);
  }
};

}  // namespace

cudaError_t launch_rmsnorm(const __nv_bfloat16* x, const __nv_bfloat16* gamma, __nv_bfloat16* y,
                           int rows, int dm, float eps, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  rmsnorm_kernel<<<rows, kNormThreads, 0, stream>>>(x, gamma, y, dm, eps);
  return cudaGetLastError();
}

}  // namespace star

namespace {
star_status lt_fail(cublasStatus_t st, const char* what) {
  char buf[256];
  snprintf(buf, sizeof buf, "cuBLASLt %s failed (status %d)", what, static_cast<int>(st));
  star::set_last_error(buf);
  return STAR_ERR_CUDA;
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

star_status star_linear(const void* x, const void* w, void* y, int M, int N, int K, int accumulate,
                        void* workspace, size_t workspace_bytes, void* cuda_stream) {
  char buf[256];
  if (M < 1 || N < 1 || K < 1 || N % 8 || K % 8 || (accumulate != 0 && accumulate != 1)) {
    snprintf(buf, sizeof buf, "bad shape M=%d N=%d K=%d (N, K multiples of 8) accumulate=%d", M,
             N, K, accumulate);
    star::set_last_error(buf);
    return STAR_ERR_INVALID_ARG;
  }
  if (!x || !w || !y || (reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w) |
                         reinterpret_cast<uintptr_t>(y)) & 15u) {
    star::set_last_error("x, w and y must be non-NULL and 16-byte aligned");
    return STAR_ERR_INVALID_ARG;
  }
  if (workspace_bytes && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))) {
    star::set_last_error("workspace must be 256-byte aligned when workspace_bytes > 0");
    return STAR_ERR_INVALID_ARG;
  }
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) {
    snprintf(buf, sizeof buf, "no CUDA device: %s", cudaGetErrorString(ce));
    star::set_last_error(buf);
    return STAR_ERR_CUDA;
  }
  cublasStatus_t st;
  {
    std::lock_guard<std::mutex> lk(star::g_lt_mu);
    if (!star::g_lt && (st = cublasLtCreate(&star::g_lt)) != CUBLAS_STATUS_SUCCESS)
      return lt_fail(st, "create");
  }
  // row-major y[M, N] = x[M, K] w[N, K]^T, read column-major, is
  // y^T (N x M) = A^T B with A = w stored K x N (ld K) and B = x stored
  // K x M (ld K); C = D = y stored N x M (ld N)
  star::LtDescs d;
  const cublasOperation_t ta = CUBLAS_OP_T, tb = CUBLAS_OP_N;
  if ((st = cublasLtMatmulDescCreate(&d.op, CUBLAS_COMPUTE_32F, CUDA_R_32F)) ||
      (st = cublasLtMatmulDescSetAttribute(d.op, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof ta)) ||
      (st = cublasLtMatmulDescSetAttribute(d.op, CUBLASLT_MATMUL_DESC_TRANSB, &tb, sizeof tb)) ||
      (st = cublasLtMatrixLayoutCreate(&d.a, CUDA_R_16BF, K, N, K)) ||
      (st = cublasLtMatrixLayoutCreate(&d.b, CUDA_R_16BF, K, M, K)) ||
      (st = cublasLtMatrixLayoutCreate(&d.c, CUDA_R_16BF, N, M, N)))
    return lt_fail(st, "descriptor");
  const star::AlgoKey key{dev, M, N, K, accumulate, workspace_bytes};
  cublasLtMatmulAlgo_t algo;
  {
    std::lock_guard<std::mutex> lk(star::g_lt_mu);
    auto it = star::g_algos.find(key);
    if (it == star::g_algos.end()) {
      cublasLtMatmulPreference_t pref = nullptr;
      cublasLtMatmulHeuristicResult_t res{};
      int nres = 0;
      st = cublasLtMatmulPreferenceCreate(&pref);
      if (st == CUBLAS_STATUS_SUCCESS)
        st = cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES,
                                                  &workspace_bytes, sizeof workspace_bytes);
      // split-K partial sums stay in fp32: no in-place reduction in the bf16
      // output (which would round every partial sum)
      const uint32_t schemes = CUBLASLT_REDUCTION_SCHEME_NONE | CUBLASLT_REDUCTION_SCHEME_COMPUTE_TYPE;
      if (st == CUBLAS_STATUS_SUCCESS)
        st = cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_REDUCTION_SCHEME_MASK,
                                                  &schemes, sizeof schemes);
      if (st == CUBLAS_STATUS_SUCCESS)
        st = cublasLtMatmulAlgoGetHeuristic(star::g_lt, d.op, d.a, d.b, d.c, d.c, pref, 1, &res,
                                            &nres);
      if (pref) cublasLtMatmulPreferenceDestroy(pref);
      if (st != CUBLAS_STATUS_SUCCESS) return lt_fail(st, "heuristic");
      if (nres < 1) return lt_fail(CUBLAS_STATUS_NOT_SUPPORTED, "heuristic (no algorithm)");
      it = star::g_algos.emplace(key, res.algo).first;
    }
    algo = it->second;
  }
  const float alpha = 1.f, beta = accumulate ? 1.f : 0.f;
  st = cublasLtMatmul(star::g_lt, d.op, &alpha, w, d.a, x, d.b, &beta, y, d.c, y, d.c, &algo,
                      workspace, workspace_bytes, static_cast<cudaStream_t>(cuda_stream));
  if (st != CUBLAS_STATUS_SUCCESS) return lt_fail(st, "matmul");
  star::set_last_error("");
  return STAR_OK;
}

}  // extern "C"
