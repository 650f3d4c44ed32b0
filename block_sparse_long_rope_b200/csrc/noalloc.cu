// star_phase2_decode_static: the Phase-2 decode step with its scratch memory
// in a fixed device array inside the library instead of a caller workspace.
//
// Who needs it: callers that may not allocate device memory themselves, for
// example a plugin whose host application owns every device allocation and
// exposes only tensors and a stream, or a latency-critical serving loop that
// must never reach cudaMalloc/cudaFree (they can block and synchronise the
// device). Such a caller passes its inputs and outputs only; the split
// counters and the per-chunk partials of the split-KV decode kernel live in
// kStaticScratchBytes (16 MiB) of device memory declared below, which every
// GPU that loads the library holds until the process exits.
//
// Contract:
//  * The array's device address is looked up once per device, on the first
//    call made with that device current (cudaGetSymbolAddress). Make that
//    first call before any stream capture.
//  * Every call on a device shares the one array and it keeps the previous
//    call's contents. The per-split chunk counters are cleared by every call;
//    everything else is fully rewritten before it is read, except the status
//    word: device errors (a bounded wait that gave up) are ORed into it and
//    stay there until star_phase2_decode_static_status reads and clears it.
//    Calls whose work overlaps on the GPU (different streams, or host
//    threads without ordering) race on the array: serialise them.
//  * Sizes that cannot fit are rejected with STAR_ERR_INVALID_ARG before
//    anything is enqueued. Nothing here allocates.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "star.h"
#include "star_common.cuh"
#include "star_kernels.cuh"

namespace {

constexpr size_t kStaticScratchBytes = 16u << 20;  // 16 MiB
constexpr int kMinChunk = 256;
constexpr int kMaxChunk = 65536;

// The scratch itself: status header and counters | chunk outputs | chunk LSEs.
static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

struct DeviceSlot {
  bool ready = false;
  void* addr = nullptr;
  int sms = 0;
};
DeviceSlot g_slots[64];
std::mutex g_slot_mu;

star_status fail_static(star_status s, const char* fmt, ...);

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Address of g_scratch on the current device (resolved once per device).
star_status scratch_address(void** out, int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_static(STAR_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail_static(STAR_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_slot_mu);
  DeviceSlot& s = g_slots[dev];
  if (!s.ready) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
      return fail_static(STAR_ERR_UNSUPPORTED, "device %d is sm_%d%d; built for sm_100a", dev, major, minor);
    cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev);
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail_static(STAR_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    s.addr = p;
    s.ready = true;
  }
  *out = s.addr;
  *sms = s.sms;
  return STAR_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// rank-3 TMA map over the head-major cache, rows [0, valid) visible, 64-row boxes
star_status cache_map(CUtensorMap* m, const void* base, int BH, int Lcap, int valid, int D) {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!fn) return fail_static(STAR_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)valid, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Lcap * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)star::kDecTile, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail_static(STAR_ERR_CUDA, "cuTensorMapEncodeTiled failed: %d", (int)r);
  return STAR_OK;
}

int chunks_per_head(int L, int b, int n, int tail_plus_T, int chunk, int* nf, int* nl, int* nt) {
  *nf = star::ceil_div(star::imin(b, L), chunk);
  *nl = star::ceil_div(L - (n - 1) * b, chunk);
  *nt = star::ceil_div(tail_plus_T, chunk);
  return (n - 1) * *nf + *nl + *nt;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace {
// Failures are reported through star_last_error, like every other entry point.
star_status fail_static(star_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  star::set_last_error(buf);
  return s;
}
}  // namespace

extern "C" {

star_status star_phase2_decode_static(const void* q, const void* k, const void* v, int T,
                                      void* k_cache, void* v_cache, int Lcap, int L,
                                      int block_len, int tail_len, float* part_o,
                                      float* part_lse, int* nsplit_out, int B, int Hq, int Hkv,
                                      int D, double theta, void* cuda_stream) {
  star::set_last_error("");
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0)
    return fail_static(STAR_ERR_INVALID_ARG, "bad head counts B=%d Hq=%d Hkv=%d", B, Hq, Hkv);
  if (D != 64 && D != 128) return fail_static(STAR_ERR_UNSUPPORTED, "head_dim %d not supported", D);
  if (T < 1 || L < 1 || block_len < 1 || tail_len < 0)
    return fail_static(STAR_ERR_INVALID_ARG, "bad T/L/block_len/tail_len");
  const int g = Hq / Hkv;
  if (T * g > star::kDecRows)
    return fail_static(STAR_ERR_INVALID_ARG,
                       "T*g = %d exceeds %d: this entry point covers decode steps only", T * g,
                       star::kDecRows);
  if ((long long)L + tail_len + T > Lcap)
    return fail_static(STAR_ERR_INVALID_ARG, "Lcap (%d) < L + tail_len + T", Lcap);
  if (!(theta > 0.0)) return fail_static(STAR_ERR_INVALID_ARG, "theta must be > 0");
  const void* ptrs[] = {q, k, v, k_cache, v_cache, part_o};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return fail_static(STAR_ERR_INVALID_ARG, "NULL or unaligned pointer");
  if (!part_lse || (reinterpret_cast<uintptr_t>(part_lse) & 3u))
    return fail_static(STAR_ERR_INVALID_ARG, "part_lse is NULL or not 4-byte aligned");

  // scratch layout and chunk size: the smallest chunk (>= 256 keys) that both
  // fits the array and leaves several CTAs per SM
  const int n = star::ceil_div(L, block_len);
  // zeroed header: status word, then one finished-chunk counter per split
  const size_t zero_bytes = star::kStatusBytes + align256((size_t)B * Hkv * (n + 1) * sizeof(int)) +
                            align256((size_t)B * Hkv * sizeof(int));
  const size_t head_bytes = zero_bytes;
  void* base = nullptr;
  int sms = 148;
  star_status st = scratch_address(&base, &sms);
  if (st != STAR_OK) return st;
  auto fits = [&](int chunk) {
    int a, b, c;
    size_t rows = (size_t)B * Hkv * chunks_per_head(L, block_len, n, tail_len + T, chunk, &a, &b, &c) *
                  star::kDecRows;
    return head_bytes + align256(rows * D * sizeof(float)) + align256(rows * sizeof(float)) <=
           kStaticScratchBytes;
  };
  // at most kMaxChunksPerSplit chunks per split (the CTA completing a split
  // reduces them), large enough to fit the array, then doubled while every
  // persistent CTA still gets several units
  const int max_split = star::imax(star::imin(block_len, L), tail_len + T);
  int chunk = kMinChunk;
  while (chunk < kMaxChunk && (star::ceil_div(max_split, chunk) > star::kMaxChunksPerSplit || !fits(chunk)))
    chunk *= 2;
  if (!fits(chunk) || star::ceil_div(max_split, chunk) > star::kMaxChunksPerSplit)
    return fail_static(STAR_ERR_INVALID_ARG,
                       "problem needs more than the %zu-byte static scratch (B=%d Hkv=%d L=%d)",
                       kStaticScratchBytes, B, Hkv, L);
  while (chunk * 2 <= kMaxChunk && chunk < max_split) {
    int a, b, c;
    long long units = (long long)B * Hkv * chunks_per_head(L, block_len, n, tail_len + T, chunk * 2, &a, &b, &c);
    if (units < 16ll * sms) break;  // keep >= 8 units per persistent CTA
    chunk *= 2;
  }

  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  unsigned char* ws = static_cast<unsigned char*>(base);
  // the counters start at zero; the status block before them is left alone
  // (sticky until star_phase2_decode_static_status)
  cudaError_t e = cudaMemsetAsync(ws + star::kStatusBytes, 0, zero_bytes - star::kStatusBytes, stream);
  if (e != cudaSuccess) return fail_static(STAR_ERR_CUDA, "counter reset: %s", cudaGetErrorString(e));

  star::DecodeParams dp;
  memset(&dp, 0, sizeof dp);
  const int valid = L + tail_len + T;
  if ((st = cache_map(&dp.tmK, k_cache, B * Hkv, Lcap, valid, D)) != STAR_OK) return st;
  if ((st = cache_map(&dp.tmV, v_cache, B * Hkv, Lcap, valid, D)) != STAR_OK) return st;
  // the decode kernel rotates q and appends the rotated k and v itself
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
  dp.ctx_pos0 = 0;
  dp.q_pos0 = L + tail_len;
  dp.with_tail = 1;
  dp.nsplit = n + 1;
  dp.chunk = chunk;
  dp.chunks_per_head = chunks_per_head(L, block_len, n, tail_len + T, chunk, &dp.nc_full,
                                       &dp.nc_last, &dp.nc_tail);
  const size_t rows = (size_t)B * Hkv * dp.chunks_per_head * star::kDecRows;
  dp.ws_o = reinterpret_cast<float*>(ws + head_bytes);
  dp.ws_lse = reinterpret_cast<float*>(ws + head_bytes + align256(rows * D * sizeof(float)));
  dp.part_o = part_o;
  dp.part_lse = part_lse;
  dp.status = reinterpret_cast<int*>(ws);
  dp.header_bytes = static_cast<int>(zero_bytes);
  dp.counters = reinterpret_cast<int*>(ws + star::kStatusBytes);
  dp.scale_ln = (float)(1.0 / sqrt((double)D));
  dp.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  e = star::launch_decode(dp, D, stream);
  if (e != cudaSuccess) return fail_static(STAR_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
  if (nsplit_out) *nsplit_out = n + 1;
  return STAR_OK;
}

star_status star_phase2_decode_static_status(void* cuda_stream) {
  star::set_last_error("");
  void* base = nullptr;
  int sms = 0;
  star_status st = scratch_address(&base, &sms);
  if (st != STAR_OK) return st;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) return fail_static(STAR_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
  int word = 0;
  e = cudaMemcpy(&word, base, sizeof word, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail_static(STAR_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
  if (word != 0) {
    e = cudaMemset(base, 0, sizeof word);
    if (e != cudaSuccess) return fail_static(STAR_ERR_CUDA, "status clear: %s", cudaGetErrorString(e));
  }
  if (word & star::kDevTimeout)
    return fail_static(STAR_ERR_DEVICE_TIMEOUT, "a decode kernel's bounded wait gave up (status 0x%x)", word);
  if (word & star::kDevBounds)
    return fail_static(STAR_ERR_DEVICE_BOUNDS, "a decode kernel found an index outside its buffer (status 0x%x)", word);
  return STAR_OK;
}

}  // extern "C"
