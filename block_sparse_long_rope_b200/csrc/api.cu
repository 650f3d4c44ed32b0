// C ABI of the Star Attention hot path (declared in include/star.h):
// argument validation, workspace layout, TMA descriptor encoding and kernel
// launches on the caller's stream. No allocation, no synchronisation (except
// star_device_status).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>

#include "star.h"
#include "star_common.cuh"
#include "star_kernels.cuh"
#include "star_plan.h"

namespace {

using star::ceil_div;
using star::chunk_subsplits;
using star::decode_chunk;
using star::decode_chunks_per_head;
using star::imin;
using star::use_decode_path;

thread_local std::string g_err;

star_status fail(star_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

star_status ok() {
  g_err.clear();
  return STAR_OK;
}

star_status cuda_fail(cudaError_t e, const char* what) {
  return fail(STAR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- device properties (cached per device) ----------------------------------
struct DevInfo {
  bool probed = false, supported = false;
  int sms = 0;
  char name[128] = {0};
};
DevInfo g_dev[64];
std::mutex g_dev_mu;

star_status check_device(int* num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(STAR_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (!d.probed) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    d.supported = (major == 10 && minor == 0);
    snprintf(d.name, sizeof d.name, "sm_%d%d", major, minor);
    d.probed = true;
  }
  if (!d.supported)
    return fail(STAR_ERR_UNSUPPORTED, "device %d is %s; this library is built for sm_100a (B200)",
                dev, d.name);
  if (num_sms) *num_sms = d.sms;
  return STAR_OK;
}

// ---- TMA descriptors ------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// rank-4 map over a token-major [B, rows, H, D] bf16 buffer; box {64, 1, 128, 1}
star_status map_token_major(CUtensorMap* m, const void* base, int B, int rows, int H, int D,
                            int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(STAR_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)rows * H * D * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(STAR_ERR_CUDA, "cuTensorMapEncodeTiled(Q) failed: %d", (int)r);
  return STAR_OK;
}

// rank-3 map over a head-major cache [B*Hkv, Lcap, D], rows [0, valid) visible;
// box {64, box_rows, 1}
star_status map_cache(CUtensorMap* m, const void* base, int BH, int Lcap, int valid, int D,
                      int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(STAR_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)valid, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Lcap * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(STAR_ERR_CUDA, "cuTensorMapEncodeTiled(cache) failed: %d", (int)r);
  return STAR_OK;
}

// ---- shared argument checks ----------------------------------------------------
star_status check_heads(int B, int Hq, int Hkv, int D) {
  if (B < 1 || Hq < 1 || Hkv < 1) return fail(STAR_ERR_INVALID_ARG, "B, Hq, Hkv must be >= 1");
  if (Hq > star::kMaxHeads)
    return fail(STAR_ERR_INVALID_ARG, "Hq (%d) must be <= %d", Hq, star::kMaxHeads);
  if (Hq % Hkv != 0) return fail(STAR_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  if (D != 64 && D != 128) return fail(STAR_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", D);
  return STAR_OK;
}

star_status check_ptr(const void* p, const char* name) {
  if (!p) return fail(STAR_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(STAR_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return STAR_OK;
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }



// Bytes of the finished-chunk counters: one per (batch, KV head, split).
size_t decode_split_counter_bytes(int B, int Hkv, int Lcap, int block_len) {
  const long long nsplit_cap = ceil_div(Lcap, block_len) + 1;
  return align_up((size_t)B * Hkv * nsplit_cap * sizeof(int));
}
// Bytes of the header of a Phase-2 workspace (zero between calls): the
// status block, the finished-chunk counters, then one finished-split counter
// per (batch, KV head).
size_t decode_header_bytes(int B, int Hkv, int Lcap, int block_len) {
  return star::kStatusBytes + decode_split_counter_bytes(B, Hkv, Lcap, block_len) +
         align_up((size_t)B * Hkv * sizeof(int));
}


// Workspace bytes of the sub-split partials of a query chunk, for the
// largest count any context of at most Lcap rows can need.
size_t chunk_scratch_bytes(int B, int T, int Hq, int Hkv, int D, int Lcap, int block_len) {
  size_t best = 0;
  for (int n = 1; (long long)n * block_len <= Lcap; ++n) {
    const int nsub = chunk_subsplits(B, Hq, Hkv, T, n * block_len, block_len, 1);
    if (nsub <= 1) continue;
    const size_t rows = (size_t)B * Hq * (n * nsub) * T;
    best = std::max(best, align_up(rows * D * sizeof(float)) + align_up(rows * sizeof(float)));
  }
  return best;
}




size_t decode_scratch_bytes(int B, int Hkv, int D, int Lcap, int block_len) {
  const long long rows = star::decode_units_bound(B, Hkv, Lcap, block_len) * star::kDecRows;
  return align_up((size_t)rows * D * sizeof(float)) + align_up((size_t)rows * sizeof(float));
}

}  // namespace

namespace star {
// Sets the calling thread's message for star_last_error (used by entry points
// defined in other files of the library).
void set_last_error(const char* msg) { g_err = msg; }

bool encode_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sms() {
  int sms = 0;
  return check_device(&sms) == STAR_OK ? sms : 0;
}

cudaError_t set_smem_attr_once(const void* fn, int slot, int dev, size_t bytes) {
  static std::atomic<bool> done[kAttrSlots][64];
  static std::mutex mu;
  const bool cacheable = slot >= 0 && slot < kAttrSlots && dev >= 0 && dev < 64;
  if (cacheable && done[slot][dev].load(std::memory_order_acquire)) return cudaSuccess;
  std::lock_guard<std::mutex> lk(mu);
  if (cacheable && done[slot][dev].load(std::memory_order_relaxed)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(bytes));
  if (e == cudaSuccess && cacheable) done[slot][dev].store(true, std::memory_order_release);
  return e;
}
}  // namespace star

extern "C" {

const char* star_last_error(void) { return g_err.c_str(); }

#ifndef STAR_BUILD_DIGEST
#define STAR_BUILD_DIGEST "unknown"
#endif
// The build digest (sources, headers, flags) ends the string, so a caller can
// check that the library it loaded was built from the sources it has.
const char* star_version(void) { return "star-b200 0.2 (sm_100a) build " STAR_BUILD_DIGEST; }

star_status star_rope(const void* x, const int64_t x_stride[3], void* y, const int64_t y_stride[3],
                      const int32_t* pos, int64_t pos0, int B, int S, int H, int D, double theta,
                      void* cuda_stream) {
  if (!x_stride || !y_stride) return fail(STAR_ERR_INVALID_ARG, "stride arrays are NULL");
  if (B < 0 || S < 0 || H < 1 || H > star::kMaxHeads)
    return fail(STAR_ERR_INVALID_ARG, "bad shape B=%d S=%d H=%d (H <= %d)", B, S, H, star::kMaxHeads);
  if (D != 64 && D != 128) return fail(STAR_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", D);
  if (!(theta > 0.0)) return fail(STAR_ERR_INVALID_ARG, "theta must be > 0");
  star_status s;
  if ((s = check_ptr(x, "x")) != STAR_OK || (s = check_ptr(y, "y")) != STAR_OK) return s;
  for (int i = 0; i < 3; ++i)
    if (x_stride[i] % 8 != 0 || y_stride[i] % 8 != 0)
      return fail(STAR_ERR_INVALID_ARG, "strides must be multiples of 8 elements");
  if (pos && (reinterpret_cast<uintptr_t>(pos) & 3u))
    return fail(STAR_ERR_INVALID_ARG, "pos is not 4-byte aligned");
  if ((s = check_device(nullptr)) != STAR_OK) return s;
  if (B == 0 || S == 0) return ok();
  star::RopeParams p{};
  p.job[0] = star::RopeJob{static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(y),
                           {x_stride[0], x_stride[1], x_stride[2]},
                           {y_stride[0], y_stride[1], y_stride[2]}, H, 1};
  p.B = B;
  p.S = S;
  p.D = D;
  p.pos = pos;
  p.pos0 = pos0;
  star::rope_set_freq(p, D, theta);
  cudaError_t e = star::launch_rope(p, 1, static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) return cuda_fail(e, "rope launch");
  return ok();
}

size_t star_phase1_workspace_bytes(int B, int L, int Hq, int D) {
  if (B < 1 || L < 1 || Hq < 1 || D < 1) return star::kStatusBytes;
  return star::kStatusBytes + align_up((size_t)B * L * Hq * D * 2);
}

size_t star_phase1_ext_workspace_bytes(int B, int L, int Hq, int Hkv, int D, int G) {
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || D < 1 || G < 0) return star::kStatusBytes;
  return star_phase1_workspace_bytes(B, L, Hq, D) + 2 * align_up((size_t)B * Hkv * G * D * 2);
}

}  // extern "C"

namespace {

// Body of star_phase1_encode / star_phase1_encode_ext. ext == false is the
// Star anchor [0, anchor_len) read in place from the cache; ext == true
// gathers the prefix table (src, pos, G rows; extra rows xk/xv) into the
// workspace and gives block i the slice bounds[i].
star_status phase1_run(const void* q, const void* k, const void* v, void* o, void* k_cache,
                       void* v_cache, int Lcap, float* lse, int B, int L, int Hq, int Hkv, int D,
                       int block_len, int anchor_len, bool ext, const int32_t* src,
                       const int32_t* pos, int G, const int32_t* bounds, const void* xk,
                       const void* xv, int NX, int ctx_pos0, double theta, void* workspace,
                       size_t workspace_bytes, void* cuda_stream, const void* qrot_in = nullptr) {
  star_status s;
  const bool prerot = qrot_in != nullptr;  // Q rotated and cache rows [0, L) filled by the caller
  if ((s = check_heads(B, Hq, Hkv, D)) != STAR_OK) return s;
  if (L < 1) return fail(STAR_ERR_INVALID_ARG, "L must be >= 1");
  if (block_len < 1) return fail(STAR_ERR_INVALID_ARG, "block_len must be >= 1");
  if (!ext && (anchor_len < 0 || anchor_len > block_len))
    return fail(STAR_ERR_INVALID_ARG, "anchor_len (%d) must lie in [0, block_len=%d]", anchor_len,
                block_len);
  if (ext) {
    if (G < 0) return fail(STAR_ERR_INVALID_ARG, "prefix table rows (%d) must be >= 0", G);
    if (NX < 0) return fail(STAR_ERR_INVALID_ARG, "extra rows (%d) must be >= 0", NX);
    if (G > 0) {
      if (!src || (reinterpret_cast<uintptr_t>(src) & 3u))
        return fail(STAR_ERR_INVALID_ARG, "prefix_src is NULL or not 4-byte aligned");
      if (!pos || (reinterpret_cast<uintptr_t>(pos) & 3u))
        return fail(STAR_ERR_INVALID_ARG, "prefix_pos is NULL or not 4-byte aligned");
      if (!bounds || (reinterpret_cast<uintptr_t>(bounds) & 3u))
        return fail(STAR_ERR_INVALID_ARG, "prefix_bounds is NULL or not 4-byte aligned");
    }
    if (NX > 0 && ((s = check_ptr(xk, "extra_k")) || (s = check_ptr(xv, "extra_v")))) return s;
    if (ctx_pos0 < 0 || (long long)ctx_pos0 + L > INT32_MAX)
      return fail(STAR_ERR_INVALID_ARG, "ctx_pos0 (%d) must be >= 0 with ctx_pos0 + L in int32",
                  ctx_pos0);
  }
  if (Lcap < L) return fail(STAR_ERR_INVALID_ARG, "Lcap (%d) < L (%d)", Lcap, L);
  if (!prerot && !(theta > 0.0)) return fail(STAR_ERR_INVALID_ARG, "theta must be > 0");
  if (prerot) {
    if ((s = check_ptr(qrot_in, "q_rot")) || (s = check_ptr(o, "o")) ||
        (s = check_ptr(k_cache, "k_cache")) || (s = check_ptr(v_cache, "v_cache")) ||
        (s = check_ptr(workspace, "workspace")))
      return s;
  } else if ((s = check_ptr(q, "q")) || (s = check_ptr(k, "k")) || (s = check_ptr(v, "v")) ||
             (s = check_ptr(o, "o")) || (s = check_ptr(k_cache, "k_cache")) ||
             (s = check_ptr(v_cache, "v_cache")) || (s = check_ptr(workspace, "workspace"))) {
    return s;
  }
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(STAR_ERR_INVALID_ARG, "lse is not 4-byte aligned");
  const size_t need = prerot ? star::kStatusBytes
                      : ext  ? star_phase1_ext_workspace_bytes(B, L, Hq, Hkv, D, G)
                             : star_phase1_workspace_bytes(B, L, Hq, D);
  if (workspace_bytes < need)
    return fail(STAR_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
  if ((long long)B * Hkv > (1ll << 31) - 1) return fail(STAR_ERR_INVALID_ARG, "B*Hkv too large");
  if ((s = check_device(nullptr)) != STAR_OK) return s;

  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  __nv_bfloat16* qrot = reinterpret_cast<__nv_bfloat16*>(ws + star::kStatusBytes);
  const size_t qrot_bytes = align_up((size_t)B * L * Hq * D * 2);
  const size_t tbl_bytes = align_up((size_t)B * Hkv * G * D * 2);
  __nv_bfloat16* pk_buf = reinterpret_cast<__nv_bfloat16*>(ws + star::kStatusBytes + qrot_bytes);
  __nv_bfloat16* pv_buf =
      reinterpret_cast<__nv_bfloat16*>(ws + star::kStatusBytes + qrot_bytes + tbl_bytes);
  cudaError_t e;

  // RoPE: Q -> workspace (token-major), K -> k_cache (head-major, rotated),
  // V -> v_cache (head-major copy). Token t sits at position t.
  star::RopeParams rp{};
  const long long qs[3] = {(long long)L * Hq * D, (long long)Hq * D, D};
  const long long ks[3] = {(long long)L * Hkv * D, (long long)Hkv * D, D};
  const long long cs[3] = {(long long)Hkv * Lcap * D, D, (long long)Lcap * D};
  rp.job[0] = star::RopeJob{static_cast<const __nv_bfloat16*>(q), qrot, {qs[0], qs[1], qs[2]},
                            {qs[0], qs[1], qs[2]}, Hq, 1};
  rp.job[1] = star::RopeJob{static_cast<const __nv_bfloat16*>(k),
                            static_cast<__nv_bfloat16*>(k_cache), {ks[0], ks[1], ks[2]},
                            {cs[0], cs[1], cs[2]}, Hkv, 1};
  rp.job[2] = star::RopeJob{static_cast<const __nv_bfloat16*>(v),
                            static_cast<__nv_bfloat16*>(v_cache), {ks[0], ks[1], ks[2]},
                            {cs[0], cs[1], cs[2]}, Hkv, 0};
  rp.B = B;
  rp.S = L;
  rp.D = D;
  rp.pos = nullptr;
  rp.pos0 = ctx_pos0;  // context row r sits at ctx_pos0 + r
  if (!prerot) {
    star::rope_set_freq(rp, D, theta);
    e = star::launch_rope(rp, 3, st);
    if (e != cudaSuccess) return cuda_fail(e, "rope launch");
  }
  if (ext && G > 0) {
    // the prefix table: K gathered and rotated at pos, V gathered, both
    // head-major [B, Hkv, G, D] in the workspace
    star::RopeParams rt{};
    const long long cs[3] = {(long long)L * Hkv * D, (long long)Hkv * D, D};
    const long long xs[3] = {(long long)NX * Hkv * D, (long long)Hkv * D, D};
    const long long ts[3] = {(long long)Hkv * G * D, D, (long long)G * D};
    rt.job[0] = star::RopeJob{static_cast<const __nv_bfloat16*>(k), pk_buf, {cs[0], cs[1], cs[2]},
                              {ts[0], ts[1], ts[2]}, Hkv, 1,
                              static_cast<const __nv_bfloat16*>(xk), {xs[0], xs[1], xs[2]}};
    rt.job[1] = star::RopeJob{static_cast<const __nv_bfloat16*>(v), pv_buf, {cs[0], cs[1], cs[2]},
                              {ts[0], ts[1], ts[2]}, Hkv, 0,
                              static_cast<const __nv_bfloat16*>(xv), {xs[0], xs[1], xs[2]}};
    rt.B = B;
    rt.S = G;
    rt.D = D;
    rt.pos = pos;
    rt.pos0 = 0;
    rt.src = src;
    rt.nsrc = L;
    rt.nx = NX;
    rt.status = reinterpret_cast<int*>(ws);
    star::rope_set_freq(rt, D, theta);
    e = star::launch_rope(rt, 2, st);
    if (e != cudaSuccess) return cuda_fail(e, "prefix table launch");
  }

  star::AttnParams ap;
  memset(&ap, 0, sizeof ap);
  if ((s = map_token_major(&ap.tmQ, prerot ? qrot_in : qrot, B, L, Hq, D)) != STAR_OK) return s;
  if ((s = map_cache(&ap.tmK, k_cache, B * Hkv, Lcap, L, D, 128)) != STAR_OK) return s;
  if ((s = map_cache(&ap.tmV, v_cache, B * Hkv, Lcap, L, D, 128)) != STAR_OK) return s;
  if (ext && G > 0) {
    if ((s = map_cache(&ap.tmKP, pk_buf, B * Hkv, G, G, D, 128)) != STAR_OK) return s;
    if ((s = map_cache(&ap.tmVP, pv_buf, B * Hkv, G, G, D, 128)) != STAR_OK) return s;
  }
  const int g = Hq / Hkv;
  ap.geom.B = B;
  ap.geom.Hq = Hq;
  ap.geom.Hkv = Hkv;
  ap.geom.hpc = (g % 2 == 0) ? 2 : 1;
  ap.geom.hps = 1;
  ap.geom.L = L;
  ap.geom.b = block_len;
  ap.geom.a = ext ? 0 : anchor_len;
  ap.geom.n = ceil_div(L, block_len);
  ap.geom.T = 0;
  ap.geom.tail_len = 0;
  ap.mode = 0;
  ap.ext = ext ? 1 : 0;
  ap.bounds = ext ? bounds : nullptr;
  ap.G = ext ? G : 0;
  const long long items = (long long)ap.geom.phase1_items();
  if (items > (1ll << 31) - 1) return fail(STAR_ERR_INVALID_ARG, "problem too large");
  ap.num_items = (int)items;
  ap.qrows = L;
  ap.nsplit = 0;
  ap.o = static_cast<__nv_bfloat16*>(o);
  ap.lse = lse;
  ap.status = reinterpret_cast<int*>(ws);
  ap.scale_ln = (float)(1.0 / sqrt((double)D));
  ap.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  e = star::launch_attn(ap, D, st);
  if (e != cudaSuccess) return cuda_fail(e, "phase-1 attention launch");
  return ok();
}

}  // namespace

extern "C" {

star_status star_phase1_encode(const void* q, const void* k, const void* v, void* o, void* k_cache,
                               void* v_cache, int Lcap, float* lse, int B, int L, int Hq, int Hkv,
                               int D, int block_len, int anchor_len, double theta, void* workspace,
                               size_t workspace_bytes, void* cuda_stream) {
  return phase1_run(q, k, v, o, k_cache, v_cache, Lcap, lse, B, L, Hq, Hkv, D, block_len,
                    anchor_len, false, nullptr, nullptr, 0, nullptr, nullptr, nullptr, 0, 0, theta,
                    workspace, workspace_bytes, cuda_stream);
}

star_status star_phase1_encode_ext(const void* q, const void* k, const void* v, void* o,
                                   void* k_cache, void* v_cache, int Lcap, float* lse, int B, int L,
                                   int Hq, int Hkv, int D, int block_len, const int32_t* prefix_src,
                                   const int32_t* prefix_pos, int G, const int32_t* prefix_bounds,
                                   const void* extra_k, const void* extra_v, int n_extra,
                                   int ctx_pos0, double theta, void* workspace,
                                   size_t workspace_bytes, void* cuda_stream) {
  return phase1_run(q, k, v, o, k_cache, v_cache, Lcap, lse, B, L, Hq, Hkv, D, block_len, 0, true,
                    prefix_src, prefix_pos, G, prefix_bounds, extra_k, extra_v, n_extra, ctx_pos0,
                    theta, workspace, workspace_bytes, cuda_stream);
}

star_status star_phase1_encode_rotated(const void* q_rot, void* o, const void* k_cache,
                                       const void* v_cache, int Lcap, float* lse, int B, int L,
                                       int Hq, int Hkv, int D, int block_len, int anchor_len,
                                       void* workspace, size_t workspace_bytes,
                                       void* cuda_stream) {
  return phase1_run(nullptr, nullptr, nullptr, o, const_cast<void*>(k_cache),
                    const_cast<void*>(v_cache), Lcap, lse, B, L, Hq, Hkv, D, block_len, anchor_len,
                    false, nullptr, nullptr, 0, nullptr, nullptr, nullptr, 0, 0, 1.0, workspace,
                    workspace_bytes, cuda_stream, q_rot);
}

size_t star_phase2_workspace_bytes(int B, int T, int Hq, int Hkv, int D, int Lcap, int block_len) {
  if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || D < 1 || Lcap < 1 || block_len < 1 || Hq % Hkv)
    return star::kStatusBytes;
  // every Phase-2 call keeps the decode header (status block and counters)
  // in front, so query-chunk and decode calls can share one workspace
  const size_t head = decode_header_bytes(B, Hkv, Lcap, block_len) + align_up((size_t)B * T * Hq * D * 2);
  if (use_decode_path(T, Hq, Hkv)) return head + decode_scratch_bytes(B, Hkv, D, Lcap, block_len);
  return head + chunk_scratch_bytes(B, T, Hq, Hkv, D, Lcap, block_len);
}

}  // extern "C"

namespace {

// Body of star_phase2_partial / star_phase2_attend / star_phase2_partial_ext;
// o_merged == NULL skips the merge. Cache row r sits at position ctx_pos0 + r,
// new token t at q_pos0 + t. with_tail == 0: context splits only, nothing
// appended (k, v unused).
star_status phase2_run(const void* q, const void* k, const void* v, int T, void* k_cache,
                       void* v_cache, int Lcap, int L, int block_len, int tail_len, int ctx_pos0,
                       int q_pos0, int with_tail, float* part_o, float* part_lse, void* o_merged,
                       float* lse_merged, int* nsplit_out, int B, int Hq, int Hkv, int D,
                       double theta, void* workspace, size_t workspace_bytes, void* cuda_stream) {
  star_status s;
  if ((s = check_heads(B, Hq, Hkv, D)) != STAR_OK) return s;
  if (T < 1) return fail(STAR_ERR_INVALID_ARG, "T must be >= 1");
  if (L < 1) return fail(STAR_ERR_INVALID_ARG, "L must be >= 1");
  if (block_len < 1) return fail(STAR_ERR_INVALID_ARG, "block_len must be >= 1");
  if (tail_len < 0) return fail(STAR_ERR_INVALID_ARG, "tail_len must be >= 0");
  if (with_tail != 0 && with_tail != 1) return fail(STAR_ERR_INVALID_ARG, "with_tail must be 0 or 1");
  if (!with_tail && tail_len != 0)
    return fail(STAR_ERR_INVALID_ARG, "tail_len must be 0 without the tail split");
  if (ctx_pos0 < 0 || q_pos0 < 0) return fail(STAR_ERR_INVALID_ARG, "positions must be >= 0");
  if (with_tail && (long long)q_pos0 != (long long)ctx_pos0 + L + tail_len)
    return fail(STAR_ERR_INVALID_ARG,
                "with the tail split the new tokens follow the cache: q_pos0 (%d) != ctx_pos0 + L "
                "+ tail_len (%lld)", q_pos0, (long long)ctx_pos0 + L + tail_len);
  if ((long long)q_pos0 + T > INT32_MAX || (long long)ctx_pos0 + Lcap > INT32_MAX)
    return fail(STAR_ERR_INVALID_ARG, "positions exceed int32");
  if ((long long)L + tail_len + (with_tail ? T : 0) > Lcap)
    return fail(STAR_ERR_INVALID_ARG, "Lcap (%d) < L + tail_len + T (%lld)", Lcap,
                (long long)L + tail_len + (with_tail ? T : 0));
  if (!(theta > 0.0)) return fail(STAR_ERR_INVALID_ARG, "theta must be > 0");
  if ((s = check_ptr(q, "q")) || (s = check_ptr(k_cache, "k_cache")) ||
      (s = check_ptr(v_cache, "v_cache")) || (s = check_ptr(part_o, "part_o")) ||
      (s = check_ptr(workspace, "workspace")))
    return s;
  if (with_tail && ((s = check_ptr(k, "k")) || (s = check_ptr(v, "v")))) return s;
  if (!part_lse || (reinterpret_cast<uintptr_t>(part_lse) & 3u))
    return fail(STAR_ERR_INVALID_ARG, "part_lse is NULL or not 4-byte aligned");
  if (o_merged && !aligned16(o_merged))
    return fail(STAR_ERR_INVALID_ARG, "o is not 16-byte aligned");
  if (lse_merged && (reinterpret_cast<uintptr_t>(lse_merged) & 3u))
    return fail(STAR_ERR_INVALID_ARG, "lse is not 4-byte aligned");
  const size_t need = star_phase2_workspace_bytes(B, T, Hq, Hkv, D, Lcap, block_len);
  if (workspace_bytes < need)
    return fail(STAR_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
  int sms = 148;
  if ((s = check_device(&sms)) != STAR_OK) return s;

  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const bool decode = use_decode_path(T, Hq, Hkv);
  // header (status block, then the decode path's split and head counters,
  // which the decode kernel returns to zero; reserved on every Phase-2 path
  // so a workspace can serve query chunks and decode steps alike), then the
  // rotated q
  const size_t header = decode_header_bytes(B, Hkv, Lcap, block_len);
  __nv_bfloat16* qrot = reinterpret_cast<__nv_bfloat16*>(ws + header);
  const size_t qrot_bytes = align_up((size_t)B * T * Hq * D * 2);
  cudaError_t e;

  // RoPE of the new tokens at positions q_pos0 + t; with the tail, K/V
  // appended to cache rows L + tail_len + t. The decode kernel does both itself.
  const int row0 = L + tail_len;
  star::RopeParams rp{};
  const long long qs[3] = {(long long)T * Hq * D, (long long)Hq * D, D};
  const long long ks[3] = {(long long)T * Hkv * D, (long long)Hkv * D, D};
  const long long cs[3] = {(long long)Hkv * Lcap * D, D, (long long)Lcap * D};
  rp.job[0] = star::RopeJob{static_cast<const __nv_bfloat16*>(q), qrot, {qs[0], qs[1], qs[2]},
                            {qs[0], qs[1], qs[2]}, Hq, 1};
  rp.job[1] = star::RopeJob{static_cast<const __nv_bfloat16*>(k),
                            static_cast<__nv_bfloat16*>(k_cache) + (size_t)row0 * D,
                            {ks[0], ks[1], ks[2]}, {cs[0], cs[1], cs[2]}, Hkv, 1};
  rp.job[2] = star::RopeJob{static_cast<const __nv_bfloat16*>(v),
                            static_cast<__nv_bfloat16*>(v_cache) + (size_t)row0 * D,
                            {ks[0], ks[1], ks[2]}, {cs[0], cs[1], cs[2]}, Hkv, 0};
  rp.B = B;
  rp.S = T;
  rp.D = D;
  rp.pos = nullptr;
  rp.pos0 = q_pos0;
  star::rope_set_freq(rp, D, theta);
  if (!decode) {
    e = star::launch_rope(rp, with_tail ? 3 : 1, st);
    if (e != cudaSuccess) return cuda_fail(e, "rope launch");
  }

  const int n = ceil_div(L, block_len);
  const int nsplit = n + with_tail;
  const int valid = L + tail_len + (with_tail ? T : 0);
  const int g = Hq / Hkv;
  if (nsplit_out) *nsplit_out = nsplit;

  if (decode) {
    star::DecodeParams dp;
    memset(&dp, 0, sizeof dp);
    if ((s = map_cache(&dp.tmK, k_cache, B * Hkv, Lcap, valid, D, star::kDecTile)) != STAR_OK) return s;
    if ((s = map_cache(&dp.tmV, v_cache, B * Hkv, Lcap, valid, D, star::kDecTile)) != STAR_OK) return s;
    dp.q_new = static_cast<const __nv_bfloat16*>(q);
    dp.k_new = static_cast<const __nv_bfloat16*>(k);
    dp.v_new = static_cast<const __nv_bfloat16*>(v);
    dp.k_cache = static_cast<__nv_bfloat16*>(k_cache);
    dp.v_cache = static_cast<__nv_bfloat16*>(v_cache);
    dp.Lcap = Lcap;
    star::rope_fill_freq(dp.inv_freq, D, theta);
    dp.B = B;
    dp.T = T;
    dp.Hq = Hq;
    dp.Hkv = Hkv;
    dp.g = g;
    dp.R = T * g;
    dp.L = L;
    dp.b = block_len;
    dp.n = n;
    dp.tail_len = tail_len;
    dp.ctx_pos0 = ctx_pos0;
    dp.q_pos0 = q_pos0;
    dp.with_tail = with_tail;
    dp.nsplit = nsplit;
    const int tail_rows = with_tail ? tail_len + T : 0;
    const int chunk = decode_chunk(B, Hkv, L, block_len, n, nsplit, tail_rows, sms);
    dp.chunk = chunk;
    dp.chunks_per_head = decode_chunks_per_head(L, block_len, n, tail_rows, chunk, &dp.nc_full,
                                                &dp.nc_last, &dp.nc_tail);
    const size_t rows = (size_t)B * Hkv * dp.chunks_per_head * star::kDecRows;
    dp.ws_o = reinterpret_cast<float*>(ws + header + qrot_bytes);
    dp.ws_lse = reinterpret_cast<float*>(ws + header + qrot_bytes + align_up(rows * D * sizeof(float)));
    dp.counters = reinterpret_cast<int*>(ws + star::kStatusBytes);
    dp.head_counters = reinterpret_cast<int*>(ws + star::kStatusBytes +
                                              decode_split_counter_bytes(B, Hkv, Lcap, block_len));
    dp.o_merged = static_cast<__nv_bfloat16*>(o_merged);
    dp.lse_merged = lse_merged;
    dp.part_o = part_o;
    dp.part_lse = part_lse;
    dp.status = reinterpret_cast<int*>(ws);
    dp.header_bytes = static_cast<int>(header);
    dp.scale_ln = (float)(1.0 / sqrt((double)D));
    dp.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    e = star::launch_decode(dp, D, st);
    if (e != cudaSuccess) return cuda_fail(e, "phase-2 decode launch");
    return ok();
  }

  star::AttnParams ap;
  memset(&ap, 0, sizeof ap);
  // chunks of at most 64 tokens put two heads in each 128-row tile
  const int hps = star::chunk_heads_per_slot(T, Hq, Hkv);
  if ((s = map_token_major(&ap.tmQ, qrot, B, T, Hq, D, 128 / hps)) != STAR_OK) return s;
  if ((s = map_cache(&ap.tmK, k_cache, B * Hkv, Lcap, valid, D, 128)) != STAR_OK) return s;
  if ((s = map_cache(&ap.tmV, v_cache, B * Hkv, Lcap, valid, D, 128)) != STAR_OK) return s;
  ap.geom.B = B;
  ap.geom.Hq = Hq;
  ap.geom.Hkv = Hkv;
  ap.geom.hpc = (g % 2 == 0) ? 2 : 1;
  ap.geom.hps = hps;
  ap.geom.L = L;
  ap.geom.b = block_len;
  ap.geom.a = 0;
  ap.geom.n = n;
  ap.geom.T = T;
  ap.geom.tail_len = tail_len;
  ap.geom.tail = with_tail;
  // Blocks cut into sub-splits: the items' partials go to the workspace and
  // one launch after the attention reduces them into part_o and, for attend,
  // merges all splits in the same pass; otherwise the items write part_o
  // directly and attend adds the plain merge.
  const int nsub = chunk_subsplits(B, Hq, Hkv, T, L, block_len, with_tail);
  ap.geom.nsub = nsub;
  ap.geom.sub_len = block_len / nsub;
  if (nsub > 1) {
    const size_t rows = (size_t)B * Hq * (n * nsub) * T;
    uint8_t* sub = ws + header + qrot_bytes;
    ap.sub_o = reinterpret_cast<float*>(sub);
    ap.sub_lse = reinterpret_cast<float*>(sub + align_up(rows * D * sizeof(float)));
  }
  ap.mode = 1;
  ap.num_items = ap.geom.phase2_items();
  ap.qrows = T;
  ap.nsplit = nsplit;
  ap.part_o = part_o;
  ap.part_lse = part_lse;
  ap.status = reinterpret_cast<int*>(ws);
  ap.scale_ln = (float)(1.0 / sqrt((double)D));
  ap.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  e = star::launch_attn(ap, D, st);
  if (e != cudaSuccess) return cuda_fail(e, "phase-2 chunk attention launch");
  if (nsub > 1) {
    e = star::launch_chunk_finish(ap.sub_o, ap.sub_lse, nsub, n, with_tail, part_o, part_lse,
                                  static_cast<__nv_bfloat16*>(o_merged), lse_merged, B, T, Hq, D,
                                  st);
    if (e != cudaSuccess) return cuda_fail(e, "sub-split reduce launch");
  } else if (o_merged) {
    star::MergeSegs segs{};
    segs.nseg = 1;
    segs.slots = nsplit;
    segs.ns[0] = nsplit;
    e = star::launch_lse_merge(part_o, part_lse, segs, static_cast<__nv_bfloat16*>(o_merged),
                               lse_merged, B, T, Hq, D, st);
    if (e != cudaSuccess) return cuda_fail(e, "lse merge launch");
  }
  return ok();
}

}  // namespace

extern "C" {

star_status star_phase2_partial(const void* q, const void* k, const void* v, int T, void* k_cache,
                                void* v_cache, int Lcap, int L, int block_len, int tail_len,
                                float* part_o, float* part_lse, int* nsplit_out, int B, int Hq,
                                int Hkv, int D, double theta, void* workspace,
                                size_t workspace_bytes, void* cuda_stream) {
  return phase2_run(q, k, v, T, k_cache, v_cache, Lcap, L, block_len, tail_len, 0, L + tail_len,
                    1, part_o, part_lse, nullptr, nullptr, nsplit_out, B, Hq, Hkv, D, theta,
                    workspace, workspace_bytes, cuda_stream);
}

star_status star_phase2_attend(const void* q, const void* k, const void* v, int T, void* k_cache,
                               void* v_cache, int Lcap, int L, int block_len, int tail_len,
                               float* part_o, float* part_lse, void* o, float* lse,
                               int* nsplit_out, int B, int Hq, int Hkv, int D, double theta,
                               void* workspace, size_t workspace_bytes, void* cuda_stream) {
  if (!o) return fail(STAR_ERR_INVALID_ARG, "o is NULL");
  return phase2_run(q, k, v, T, k_cache, v_cache, Lcap, L, block_len, tail_len, 0, L + tail_len,
                    1, part_o, part_lse, o, lse, nsplit_out, B, Hq, Hkv, D, theta, workspace,
                    workspace_bytes, cuda_stream);
}

star_status star_phase2_partial_ext(const void* q, const void* k, const void* v, int T,
                                    void* k_cache, void* v_cache, int Lcap, int L, int block_len,
                                    int tail_len, int ctx_pos0, int q_pos0, int with_tail,
                                    float* part_o, float* part_lse, int* nsplit_out, int B, int Hq,
                                    int Hkv, int D, double theta, void* workspace,
                                    size_t workspace_bytes, void* cuda_stream) {
  return phase2_run(q, k, v, T, k_cache, v_cache, Lcap, L, block_len, tail_len, ctx_pos0, q_pos0,
                    with_tail, part_o, part_lse, nullptr, nullptr, nsplit_out, B, Hq, Hkv, D,
                    theta, workspace, workspace_bytes, cuda_stream);
}

star_status star_lse_merge(const float* part_o, const float* part_lse, int nsplit, void* o,
                           float* lse, int B, int T, int Hq, int D, void* cuda_stream) {
  if (nsplit < 1 || B < 1 || T < 1 || Hq < 1)
    return fail(STAR_ERR_INVALID_ARG, "bad shape nsplit=%d B=%d T=%d Hq=%d", nsplit, B, T, Hq);
  if (D != 64 && D != 128) return fail(STAR_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", D);
  star_status s;
  if ((s = check_ptr(part_o, "part_o")) || (s = check_ptr(o, "o"))) return s;
  if (!part_lse || (reinterpret_cast<uintptr_t>(part_lse) & 3u))
    return fail(STAR_ERR_INVALID_ARG, "part_lse is NULL or not 4-byte aligned");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(STAR_ERR_INVALID_ARG, "lse is not 4-byte aligned");
  if ((s = check_device(nullptr)) != STAR_OK) return s;
  star::MergeSegs segs{};
  segs.nseg = 1;
  segs.slots = nsplit;
  segs.ns[0] = nsplit;
  cudaError_t e = star::launch_lse_merge(part_o, part_lse, segs, static_cast<__nv_bfloat16*>(o),
                                         lse, B, T, Hq, D, static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) return cuda_fail(e, "lse merge launch");
  return ok();
}

star_status star_lse_merge_ranks(const float* part_o, const float* part_lse, int nranks,
                                 const int* nsplit_of_rank, int nsplit_stride, void* o, float* lse,
                                 int B, int T, int Hq, int D, void* cuda_stream) {
  if (nranks < 1 || nranks > star::kMaxMergeSegs)
    return fail(STAR_ERR_INVALID_ARG, "nranks (%d) must lie in [1, %d]", nranks,
                star::kMaxMergeSegs);
  if (!nsplit_of_rank) return fail(STAR_ERR_INVALID_ARG, "nsplit_of_rank is NULL");
  if (nsplit_stride < 1 || B < 1 || T < 1 || Hq < 1)
    return fail(STAR_ERR_INVALID_ARG, "bad shape stride=%d B=%d T=%d Hq=%d", nsplit_stride, B, T,
                Hq);
  if (D != 64 && D != 128) return fail(STAR_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", D);
  star::MergeSegs segs{};
  segs.nseg = nranks;
  segs.slots = nsplit_stride;
  long long total = 0;
  for (int r = 0; r < nranks; ++r) {
    if (nsplit_of_rank[r] < 0 || nsplit_of_rank[r] > nsplit_stride)
      return fail(STAR_ERR_INVALID_ARG, "rank %d has %d splits (stride %d)", r, nsplit_of_rank[r],
                  nsplit_stride);
    segs.ns[r] = nsplit_of_rank[r];
    total += nsplit_of_rank[r];
  }
  if (total < 1) return fail(STAR_ERR_INVALID_ARG, "no splits to merge");
  star_status s;
  if ((s = check_ptr(part_o, "part_o")) || (s = check_ptr(o, "o"))) return s;
  if (!part_lse || (reinterpret_cast<uintptr_t>(part_lse) & 3u))
    return fail(STAR_ERR_INVALID_ARG, "part_lse is NULL or not 4-byte aligned");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(STAR_ERR_INVALID_ARG, "lse is not 4-byte aligned");
  if ((s = check_device(nullptr)) != STAR_OK) return s;
  cudaError_t e = star::launch_lse_merge(part_o, part_lse, segs, static_cast<__nv_bfloat16*>(o),
                                         lse, B, T, Hq, D, static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) return cuda_fail(e, "lse merge launch");
  return ok();
}

star_status star_device_status(void* workspace, void* cuda_stream) {
  if (!workspace) return fail(STAR_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  // word 0: the status bits (sticky until read here); word 1: the size of the
  // header the last decode call counted in, cleared with the status after an
  // error (an aborted call may leave its counters non-zero)
  int words[2] = {0, 0};
  e = cudaMemcpy(words, workspace, sizeof words, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  const int word = words[0];
  if (word != 0) {
    const size_t clear = std::max<size_t>(sizeof word, static_cast<size_t>(std::max(words[1], 0)));
    e = cudaMemset(workspace, 0, clear);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
  }
  if (word & star::kDevTimeout)
    return fail(STAR_ERR_DEVICE_TIMEOUT, "a kernel's bounded wait gave up (status 0x%x)", word);
  if (word & star::kDevBounds)
    return fail(STAR_ERR_DEVICE_BOUNDS, "a kernel found an index outside its buffer (status 0x%x)", word);
  return ok();
}

star_status star_debug_wait_probe(void* workspace, double seconds, void* cuda_stream) {
  star_status s;
  if ((s = check_ptr(workspace, "workspace")) != STAR_OK) return s;
  if (!(seconds > 0.0) || seconds > 2.0)
    return fail(STAR_ERR_INVALID_ARG, "seconds must lie in (0, 2]");
  if ((s = check_device(nullptr)) != STAR_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, star::kStatusBytes, st);
  if (e != cudaSuccess) return cuda_fail(e, "status reset");
  e = star::launch_debug_wait_probe(static_cast<int*>(workspace),
                                    static_cast<unsigned long long>(seconds * 1e9), st);
  if (e != cudaSuccess) return cuda_fail(e, "wait probe launch");
  return ok();
}

star_status star_debug_index(int L, int block_len, int anchor_len, int32_t* blk, int32_t* pos,
                             int32_t* kv_ranges, void* cuda_stream) {
  if (L < 1 || block_len < 1 || anchor_len < 0 || anchor_len > block_len)
    return fail(STAR_ERR_INVALID_ARG, "bad L/block_len/anchor_len");
  star_status s;
  if ((s = check_ptr(blk, "blk")) || (s = check_ptr(pos, "pos")) || (s = check_ptr(kv_ranges, "kv_ranges")))
    return s;
  if ((s = check_device(nullptr)) != STAR_OK) return s;
  cudaError_t e = star::launch_debug_index(L, block_len, anchor_len, blk, pos, kv_ranges,
                                           static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) return cuda_fail(e, "debug index launch");
  return ok();
}

}  // extern "C"
