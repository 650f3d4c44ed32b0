// Parameter blocks and launchers of the Star Attention kernels (internal to
// the library; the public surface is include/star.h).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "star_index.cuh"

namespace star {

// ---- RoPE / cache write ----------------------------------------------------
constexpr int kMaxHeads = 2048;  // heads per call (keeps the RoPE kernel's unit index math in 32 bits)
struct RopeJob {
  const __nv_bfloat16* x;
  __nv_bfloat16* y;
  long long xs[3];  // element strides of (B, S, H); D is contiguous
  long long ys[3];
  int H;
  int rotate;       // 0: plain copy (V into the cache)
  const __nv_bfloat16* x2;  // gather mode: the given rows [B, nx, H, D]
  long long x2s[3];
};
struct RopeParams {
  RopeJob job[3];
  int B, S, D;
  int tpc;             // tokens per CTA (1..kRopeMaxTok; launch_rope picks it when 0)
  const int32_t* pos;  // nullable: position of token s is pos0 + s
  long long pos0;
  // gather mode (src != nullptr): output token s reads row src[s] of x when
  // 0 <= src[s] < nsrc, row -1 - src[s] of x2 when -nx <= src[s] < 0;
  // any other index writes a zero row and sets kDevBounds in *status
  const int32_t* src;
  int nsrc, nx;
  int* status;
  double inv_freq[64];  // theta^(-2i/D), i < D/2 (fp64, from the host)
};
constexpr int kRopeMaxTok = 8;
// Fills out[0..63] with theta^(-2i/D) for i < D/2 (zero beyond).
void rope_fill_freq(double* out, int D, double theta);
inline void rope_set_freq(RopeParams& p, int D, double theta) { rope_fill_freq(p.inv_freq, D, theta); }
cudaError_t launch_rope(const RopeParams& p, int njobs, cudaStream_t stream);

// ---- tcgen05 attention (Phase 1, and Phase 2 query chunks) -----------------
struct AttnParams {
  CUtensorMap tmQ;  // rotated Q [B, rows, Hq, D]: dims {D, Hq, rows, B}, box {64, 1, 128, 1}
  CUtensorMap tmK;  // K cache [B*Hkv, Lvalid, D]: dims {D, Lvalid, B*Hkv}, box {64, 128, 1}
  CUtensorMap tmV;  // V cache, same shape as K
  CUtensorMap tmKP;  // prefix table K (rotated) [B*Hkv, G, D] (ext mode, G > 0)
  CUtensorMap tmVP;  // prefix table V
  int ext;           // Phase 1 with a gathered prefix table (star_phase1_encode_ext)
  const int32_t* bounds;  // device [n][2]: block i sees table rows [bounds[2i], bounds[2i+1])
  int G;                  // prefix table rows
  AttnGeom geom;
  int mode;         // 0: Phase 1 (bf16 o, lse), 1: Phase 2 partials
  int num_items;
  int qrows;        // rows per (batch, head) in the rotated-Q buffer
  int nsplit;
  __nv_bfloat16* o;  // Phase 1: [B, L, Hq, D]
  float* lse;        // Phase 1: [B, Hq, L] (nullable)
  float* part_o;     // Phase 2: [B, Hq, nsplit, T, D], nsplit = n + tail (the API's splits)
  float* part_lse;   // Phase 2: [B, Hq, nsplit, T]
  // Phase-2 query chunks whose blocks are cut into nsub sub-splits: the
  // items' partials go to sub_o / sub_lse ([B, Hq, n * nsub, T, D] / [.., T]),
  // which launch_chunk_finish reduces into part_o.
  float* sub_o;
  float* sub_lse;
  int* status;
  float scale_log2;  // log2(e) / sqrt(D)
  float scale_ln;    // 1 / sqrt(D)
};
size_t attn_smem_bytes(int D);
cudaError_t launch_attn(const AttnParams& p, int D, cudaStream_t stream);

// ---- Phase 2 decode (split-KV, HBM-bound) ----------------------------------
constexpr int kDecRows = 16;   // (token, head) rows per CTA: one mma.sync M tile
constexpr int kDecTile = 64;   // keys per staged K/V tile
constexpr int kMaxChunksPerSplit = 64;  // chunk size is chosen so a split has at most this many
struct DecodeParams {
  CUtensorMap tmK;  // K cache: dims {D, Lvalid, B*Hkv}, box {64, 64, 1}
  CUtensorMap tmV;
  const __nv_bfloat16* q_new;  // pre-RoPE q of the new tokens [B, T, Hq, D]
  const __nv_bfloat16* k_new;  // pre-RoPE k [B, T, Hkv, D], appended to the cache in-kernel
  const __nv_bfloat16* v_new;  // v [B, T, Hkv, D]
  __nv_bfloat16* k_cache;      // [B*Hkv, Lcap, D]
  __nv_bfloat16* v_cache;
  int Lcap;
  double inv_freq[64];         // theta^(-2i/D), i < D/2
  int B, T, Hq, Hkv, g, R;  // R = T * g rows (<= kDecRows)
  int L, b, n, tail_len;    // context, block length, context splits, earlier tail tokens
  int ctx_pos0;             // position of cache row 0 (row r sits at ctx_pos0 + r)
  int q_pos0;               // position of new token 0
  int with_tail;            // 1: append the new tokens and attend the tail split
  int nsplit;               // n + with_tail
  int chunk;                // keys per CTA (multiple of kDecTile)
  int nc_full, nc_last, nc_tail, chunks_per_head;  // chunk counts per split kind
  float* ws_o;     // [B*Hkv, chunks_per_head, kDecRows, D] chunk-normalised output
  float* ws_lse;   // [B*Hkv, chunks_per_head, kDecRows]
  int* counters;   // [B*Hkv, nsplit] finished chunks per split; zero between calls
  int* head_counters;  // [B*Hkv] finished splits per (batch, KV head); zero between calls
  __nv_bfloat16* o_merged;  // nullable: [B, T, Hq, D] merged output (also needs head_counters)
  float* lse_merged;        // nullable: [B, Hq, T]
  float* part_o;   // [B, Hq, nsplit, T, D]
  float* part_lse; // [B, Hq, nsplit, T]
  int* status;            // status word; status[1] receives header_bytes
  int header_bytes;       // workspace bytes holding the status block and the counters
  float scale_log2, scale_ln;
};
size_t decode_smem_bytes(int D);
cudaError_t launch_decode(const DecodeParams& p, int D, cudaStream_t stream);

// ---- LSE merge ---------------------------------------------------------------
// Partials in `nseg` segments (e.g. one per rank after an all-gather):
// segment s starts at split row s * B * Hq * slots and holds its ns[s] <=
// slots splits laid out densely, [B, Hq, ns[s], T, D] / [B, Hq, ns[s], T].
constexpr int kMaxMergeSegs = 64;
struct MergeSegs {
  int nseg, slots;
  int ns[kMaxMergeSegs];
};
cudaError_t launch_lse_merge(const float* part_o, const float* part_lse, const MergeSegs& segs,
                             __nv_bfloat16* o, float* lse, int B, int T, int Hq, int D,
                             cudaStream_t stream);
// After a query chunk whose n context blocks were cut into nsub sub-splits
// (sub_o / sub_lse [B, Hq, n * nsub, T, D] / [.., T]): reduces each block's
// sub-splits into part_o / part_lse [B, Hq, n + tail, T, (D)] (the tail
// split is already there) and, when o is not NULL, merges all n + tail
// splits into o [B, T, Hq, D] / lse [B, Hq, T] in the same pass.
cudaError_t launch_chunk_finish(const float* sub_o, const float* sub_lse, int nsub, int n,
                                int tail, float* part_o, float* part_lse, __nv_bfloat16* o,
                                float* lse, int B, int T, int Hq, int D, cudaStream_t stream);

// ---- projection GEMM (tcgen05): y[M, N] = x[M, K] w[N, K]^T with epilogues --
struct GemmParams {
  CUtensorMap tmA;  // x [M, K] row-major: dims {K, M}, box {64, 128}
  CUtensorMap tmB;  // w [N, K] row-major: dims {K, N}, box {64, 256}
  int M, N, K;
  int m_tiles, n_tiles, k_blocks;  // 128-row, 256-column and 64-deep tiles
  __nv_bfloat16* y;
  int accumulate;   // 1: y = bf16(y + bf16(acc)) (row-major, no rotation)
  int rd;           // 64 / 128: rotate every rd-column head (RoPE); 0: no rotation
  int hd;           // head dim of the cache layout (cache_rows > 0)
  int seq_len;      // rows per sequence: row m is token m % seq_len of sequence m / seq_len
  int cache_rows;   // 0: y row-major [M, N]; > 0: y head-major [M / seq_len, N / hd, cache_rows, hd]
  long long pos0;   // RoPE position of token t = pos0 + t
  double inv_freq[64];  // theta^(-2i/rd), i < rd/2
  const float2* rope_tab;  // [seq_len][rd/2] fp32 roundings of (cos, sin)(pos * inv_freq)
  // K and V in one GEMM: columns n >= n_split go, unrotated, to y2 as its
  // column n - n_split (same layout as y); n_split = N otherwise
  int n_split;
  __nv_bfloat16* y2;
  int* status;      // device status word (bounded waits)
};
size_t gemm_smem_bytes();
cudaError_t launch_gemm(const GemmParams& p, int sms, cudaStream_t stream);
// Fills tab[t][i] = fp32 roundings of the fp64 (cos, sin) of (pos0 + t) *
// inv_freq[i] (rope_angle), t < S, i < half.
cudaError_t launch_rope_table(float2* tab, int S, int half, long long pos0, const double* inv_freq,
                              cudaStream_t stream);

// ---- error message of the calling thread (star_last_error) -------------------
void set_last_error(const char* msg);

// ---- per-device launch set-up ---------------------------------------------------
// Raises kernel `fn`'s dynamic shared-memory limit to `bytes` on device `dev`
// the first time it is asked for that (slot, device); later calls return at
// once. Safe to call from several host threads. slot < kAttrSlots names the
// kernel (one slot per kernel instantiation).
constexpr int kAttrSlots = 16;  // attention 0-3, GEMM 4-6, decode 8-9
cudaError_t set_smem_attr_once(const void* fn, int slot, int dev, size_t bytes);
// Rank-2 TMA map of a row-major bf16 matrix (inner x outer elements, rows
// row_bytes apart) with a box of box_inner x box_outer and 128-byte swizzle;
// false if the driver rejects it.
bool encode_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);
// SM count of the current device if it is supported (sm_100), else 0 (the
// message is then set for star_last_error).
int device_sms();

// ---- debug: device-evaluated index math --------------------------------------
cudaError_t launch_debug_index(int L, int b, int a, int32_t* blk, int32_t* pos, int32_t* ranges,
                               cudaStream_t stream);
cudaError_t launch_debug_wait_probe(int* status, unsigned long long limit_ns, cudaStream_t stream);

}  // namespace star
