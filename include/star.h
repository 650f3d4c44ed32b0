/*
 * star.h — C ABI of the Star Attention hot path for NVIDIA B200 (sm_100a).
 *
 * Star Attention (arXiv 2411.17116) encodes a long context in two phases:
 *   Phase 1  the context is split into blocks c_1..c_n of b tokens; every
 *            block i >= 2 is prefixed with the anchor block c_1, which keeps
 *            its original position IDs, and attends causally only inside that
 *            augmented block; the anchor's KV entries are then dropped
 *            [pith 2WVXFXZ2, "What carries the argument"; minor comment on
 *            Section 2.1: c'_1 = c_1 has b tokens, only blocks i >= 2 carry
 *            the anchor].
 *   Phase 2  query and generated tokens attend to every cached token: each
 *            block ("host") returns a local attention output and a softmax
 *            statistic, and the query side re-weights them into exact
 *            global attention [pith 2WVXFXZ2, Referee summary; Circularity
 *            check; minor comment on Algorithm 2: weight exp(s_h - s_global)].
 * On one GPU the pages' hosts become blocks processed in parallel.
 *
 * Conventions shared by every call
 *   - Memory is owned by the caller (device pointers unless stated). The
 *     library allocates nothing and keeps no state besides a thread-local
 *     error message and per-device properties it caches on first use.
 *   - Every call is asynchronous on `cuda_stream` (a cudaStream_t; NULL is
 *     the legacy default stream). None synchronises, except
 *     star_device_status.
 *   - Arguments are validated before anything is launched; on a non-OK
 *     status nothing was enqueued (except STAR_ERR_CUDA from a launch).
 *   - Element types: bf16 for Q/K/V/O and the KV cache, fp32 for LSE and
 *     partials. LSE values are natural logarithms.
 *   - Softmax scale 1/sqrt(D). Query head h uses KV head h / (Hq / Hkv)
 *     (contiguous GQA groups).
 *   - RoPE is rotate-half with base theta: pair (x_i, x_{i+D/2}) turns by the
 *     angle p * theta^(-2i/D); token t of the context sits at position t, so
 *     the anchor keeps positions 0..a-1 in every block.
 *   - Supported head_dim D: 64 and 128; at most 2048 heads. Pointers must be
 *     16-byte aligned.
 *   - Device errors found inside kernels (a bounded wait that gave up, an
 *     index outside its buffer) are recorded in a status word at the start of
 *     the call's workspace and read back by star_device_status.
 *   - A workspace must be zero-filled once before its first use. After that
 *     the library keeps it consistent: status bits are sticky (calls OR them
 *     in, only star_device_status reads and clears them), and the counters of
 *     the decode path, which every Phase-2 call keeps at the start of its
 *     workspace, return to zero at the end of every call (after a device
 *     error star_device_status clears them too). A workspace that decode
 *     calls use may be shared with other Phase-2 calls of the same B, Hkv,
 *     Lcap and block_len; before any other reuse it must be zero-filled
 *     again. No call resets the workspace, so consecutive decode kernels run
 *     back to back: the decode kernel is launched as a programmatic dependent
 *     launch and may start while the previous kernel in the stream drains.
 *     It streams cache rows [0, L) at once and waits for that kernel to end
 *     before it reads q, k or v, touches the tail rows, or writes anything.
 *     Cache rows [0, L) must therefore not be written by the kernel launched
 *     just before a decode call (Phase 1 never is: its last kernel only reads
 *     the cache), and consecutive decode calls on one cache keep the context
 *     length L and grow only the tail. This is how Phase 2 proceeds: the
 *     context is fixed after Phase 1.
 */
#ifndef STAR_H_
#define STAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  STAR_OK = 0,
  STAR_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or shape */
  STAR_ERR_UNSUPPORTED = 2,   /* head_dim or device not supported */
  STAR_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
  STAR_ERR_DEVICE_TIMEOUT = 4,/* a kernel's bounded wait gave up */
  STAR_ERR_DEVICE_BOUNDS = 5  /* a kernel found an index outside its buffer */
} star_status;

/* Message describing the calling thread's last non-OK status ("" if none).
 * The pointer stays valid until the next call on the same thread. */
const char* star_last_error(void);

/* Library version string; it ends with the digest of the sources, headers and
 * build flags the library was built from. */
const char* star_version(void);

/*
 * star_rope — rotate-half RoPE at given positions
 * [pith 2607.20457, "What carries the argument": original global position
 * IDs preserve RoPE distances; pith 2WVXFXZ2: the anchor keeps c_1's
 * original positional indices].
 *
 *   y[b,s,h,:] = RoPE(x[b,s,h,:], p_s),  p_s = pos[s] if pos != NULL else pos0 + s
 *
 * x, y: bf16, D contiguous; x_stride / y_stride give the element strides of
 * the (B, S, H) dimensions (each a multiple of 8). x and y may be the same
 * buffer (in place) but must not otherwise overlap. pos: device int32[S] or
 * NULL. Angles, their reduction modulo 2*pi and sine/cosine are fp64; y is
 * the correctly rounded bf16 (nearest even) of the exact rotation.
 */
star_status star_rope(const void* x, const int64_t x_stride[3], void* y,
                      const int64_t y_stride[3], const int32_t* pos, int64_t pos0, int B,
                      int S, int H, int D, double theta, void* cuda_stream);

/* Workspace bytes star_phase1_encode needs: the rotated Q (bf16
 * [B, L, Hq, D]) plus a 256-byte status header. */
size_t star_phase1_workspace_bytes(int B, int L, int Hq, int D);

/*
 * star_phase1_encode — Phase 1, anchor-block blockwise-local causal encoding
 * [pith 2WVXFXZ2, "What carries the argument"; minor comment on
 * Section 2.1; abstract: "the context is processed using blockwise-local
 * attention ... in parallel"].
 *
 * Inputs (pre-RoPE, token-major): q[B, L, Hq, D], k/v[B, L, Hkv, D].
 * Row r of block i = r / block_len attends to
 *   i == 0 : keys [0, r]                       (c'_1 = c_1, plain causal)
 *   i >= 1 : keys [0, anchor_len) U [i*block_len, r]
 * The anchor's keys are block 1's cache rows (same tokens, same positions),
 * so they are computed once and shared; no anchor copy is ever stored.
 * Outputs:
 *   o[B, L, Hq, D]             bf16, softmax-normalised
 *   k_cache/v_cache[B, Hkv, Lcap, D]  rows [0, L) written: K rotated, V copied
 *                              (head-major; rows >= L untouched)
 *   lse[B, Hq, L]              fp32 natural-log statistic, or NULL
 * anchor_len in [0, block_len]; 0 disables the anchor (the pages' "no
 * anchor" ablation); block_len >= L gives full causal attention.
 * Requires Lcap >= L, workspace_bytes >= star_phase1_workspace_bytes().
 */
star_status star_phase1_encode(const void* q, const void* k, const void* v, void* o,
                               void* k_cache, void* v_cache, int Lcap, float* lse, int B, int L,
                               int Hq, int Hkv, int D, int block_len, int anchor_len,
                               double theta, void* workspace, size_t workspace_bytes,
                               void* cuda_stream);

/*
 * star_phase1_encode_rotated — star_phase1_encode when the caller has already
 * rotated Q and written the cache (for example with star_linear_rope):
 * q_rot[B, L, Hq, D] holds RoPE'd queries at positions 0..L-1 and
 * k_cache/v_cache[B, Hkv, Lcap, D] rows [0, L) hold the rotated keys and the
 * values. Only the block-sparse attention runs; the visibility rule, o and
 * lse are those of star_phase1_encode. workspace: >= 256 bytes (the status
 * word), zero-filled once. Errors as star_phase1_encode.
 */
star_status star_phase1_encode_rotated(const void* q_rot, void* o, const void* k_cache,
                                       const void* v_cache, int Lcap, float* lse, int B, int L,
                                       int Hq, int Hkv, int D, int block_len, int anchor_len,
                                       void* workspace, size_t workspace_bytes,
                                       void* cuda_stream);

/* Workspace bytes star_phase1_encode_ext needs for a prefix table of G
 * rows: as star_phase1_encode plus the table's rotated K and its V (bf16
 * [B, Hkv, G, D] each). */
size_t star_phase1_ext_workspace_bytes(int B, int L, int Hq, int Hkv, int D, int G);

/*
 * star_phase1_encode_ext — Phase 1 with a generalised prefix. Instead of the
 * anchor of star_phase1_encode, every block sees a slice of one gathered
 * prefix table of G rows:
 *   table row g  = context row prefix_src[g] of k/v when prefix_src[g] >= 0,
 *                  row -1 - prefix_src[g] of extra_k/extra_v otherwise; its
 *                  key is rotated at position prefix_pos[g];
 *   block i sees table rows [prefix_bounds[2i], prefix_bounds[2i+1]), all
 *                  visible, then its own rows causally at their own positions.
 * This covers the Star anchor (rows 0..a-1 at positions 0..a-1, blocks i >= 1
 * see [0, a)) [pith 2WVXFXZ2, "What carries the argument"]; the anchor
 * ablations — no anchor, anchor position IDs moved or randomised, anchor
 * content replaced (atlas.scime.ai summary, measured-effects table); and
 * Pulsar's [sink || Sigma_0 || ... || Sigma_{i-1} || B_i] with every row at
 * its original global position, one table of which block i sees a leading
 * part [pith 2607.20457, "What carries the argument"]. A row listed twice
 * counts twice; block 0 takes its slice too.
 *
 * prefix_src, prefix_pos : device int32 [G]; prefix_bounds: device int32
 *   [n][2], n = ceil(L / block_len). All three may be NULL when G == 0.
 * extra_k, extra_v : device bf16 [B, n_extra, Hkv, D] pre-RoPE, 16-byte
 *   aligned; NULL when n_extra == 0.
 * ctx_pos0 : position of context row 0 (row r of q/k/v sits at ctx_pos0 + r;
 *   0 for a whole sequence). A shard of a sequence split by blocks over
 *   several GPUs passes the global position of its first row, with the
 *   anchor as given rows at positions 0..a-1 [pith 2WVXFXZ2, "What carries
 *   the argument": every host gets the anchor block with its original
 *   positions]. Block boundaries are counted from row 0 of the call.
 * Other arguments, the outputs and the KV cache as for star_phase1_encode.
 * Errors: invalid arguments as for star_phase1_encode (STAR_ERR_INVALID_ARG,
 *   nothing launched). A prefix_src outside [-n_extra, L) gives a zero row; a
 *   slice outside [0, G] (or reversed) is clamped to it; either records
 *   STAR_ERR_DEVICE_BOUNDS in the workspace status word (star_device_status).
 */
star_status star_phase1_encode_ext(const void* q, const void* k, const void* v, void* o,
                                   void* k_cache, void* v_cache, int Lcap, float* lse, int B, int L,
                                   int Hq, int Hkv, int D, int block_len, const int32_t* prefix_src,
                                   const int32_t* prefix_pos, int G, const int32_t* prefix_bounds,
                                   const void* extra_k, const void* extra_v, int n_extra,
                                   int ctx_pos0, double theta, void* workspace,
                                   size_t workspace_bytes, void* cuda_stream);

/* Workspace bytes star_phase2_partial needs for up to T new tokens with a
 * cache of capacity Lcap (context L plus tail) split into blocks of
 * block_len: the header (256-byte status block, then the decode path's
 * split and head counters, kept on every Phase-2 path), the rotated q and,
 * on the decode path (T * Hq / Hkv <= 16), the chunk partials. */
size_t star_phase2_workspace_bytes(int B, int T, int Hq, int Hkv, int D, int Lcap, int block_len);

/*
 * star_phase2_partial — Phase 2 per-block partial attention
 * [pith 2WVXFXZ2, Referee summary: the query is broadcast and each host
 * computes local softmax statistics; abstract: query and response tokens
 * attend to all prior cached tokens].
 *
 * T new tokens (a query chunk, or one decode token) with pre-RoPE
 * q[B, T, Hq, D], k/v[B, T, Hkv, D] sit at positions L + tail_len + t. The
 * call rotates q and k, appends k/v into cache rows L + tail_len + t, then
 * for every split writes the split-local softmax-normalised output and its
 * LSE:
 *   split j < n (n = ceil(L / block_len)): context block j, keys
 *                 [j*block_len, min((j+1)*block_len, L)), all visible
 *   split n (tail): cache rows [L, L + tail_len + t], causal per token
 *   part_o[B, Hq, n+1, T, D] fp32, part_lse[B, Hq, n+1, T] fp32
 * *nsplit_out (host int, may be NULL) receives n + 1.
 * Requires Lcap >= L + tail_len + T and cache rows [0, L + tail_len) filled
 * by earlier calls; workspace_bytes >= star_phase2_workspace_bytes().
 */
star_status star_phase2_partial(const void* q, const void* k, const void* v, int T, void* k_cache,
                                void* v_cache, int Lcap, int L, int block_len, int tail_len,
                                float* part_o, float* part_lse, int* nsplit_out, int B, int Hq,
                                int Hkv, int D, double theta, void* workspace,
                                size_t workspace_bytes, void* cuda_stream);

/*
 * star_phase2_attend — star_phase2_partial followed by the exact merge of its
 * partials (as star_lse_merge) in the same call [pith 2WVXFXZ2, Referee
 * summary; minor comment on Algorithm 2]. part_o / part_lse are written as
 * by star_phase2_partial; o[B, T, Hq, D] bf16 (required) and lse[B, Hq, T]
 * fp32 (nullable) receive the merged global attention. On the decode path
 * (T * Hq / Hkv <= 16) the merge runs inside the decode kernel: the last CTA
 * to finish the splits of a (batch, KV head) merges them, so no extra launch
 * is made. Workspace as for star_phase2_partial.
 */
star_status star_phase2_attend(const void* q, const void* k, const void* v, int T, void* k_cache,
                               void* v_cache, int Lcap, int L, int block_len, int tail_len,
                               float* part_o, float* part_lse, void* o, float* lse,
                               int* nsplit_out, int B, int Hq, int Hkv, int D, double theta,
                               void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * star_phase2_partial_ext — star_phase2_partial for one shard of a sequence
 * whose context blocks are spread over several GPUs [pith 2WVXFXZ2, Referee
 * summary: the query is broadcast, every host computes a local attention
 * output and softmax statistic over its own KV cache, the query host
 * re-weights them; "What carries the argument": KV caches never move].
 *   cache row r (r < L + tail_len) sits at position ctx_pos0 + r;
 *   new token t is rotated at position q_pos0 + t;
 *   with_tail = 1 (the query host): as star_phase2_partial — the new tokens'
 *     k/v are rotated and appended at cache rows L + tail_len + t, which
 *     requires q_pos0 == ctx_pos0 + L + tail_len, and split n is the causal
 *     tail; nsplit = n + 1;
 *   with_tail = 0 (any other host): context splits only; k and v are unused
 *     (may be NULL), tail_len must be 0, nothing is written to the cache;
 *     nsplit = n.
 * n = ceil(L / block_len) counts the shard's own blocks. part_o [B, Hq,
 * nsplit, T, D] and part_lse [B, Hq, nsplit, T] fp32 as star_phase2_partial.
 * Workspace: star_phase2_workspace_bytes(B, T, Hq, Hkv, D, Lcap, block_len).
 * Errors: STAR_ERR_INVALID_ARG for negative positions, with_tail not 0/1,
 * q_pos0 inconsistent with the tail, or positions past int32.
 */
star_status star_phase2_partial_ext(const void* q, const void* k, const void* v, int T,
                                    void* k_cache, void* v_cache, int Lcap, int L, int block_len,
                                    int tail_len, int ctx_pos0, int q_pos0, int with_tail,
                                    float* part_o, float* part_lse, int* nsplit_out, int B, int Hq,
                                    int Hkv, int D, double theta, void* workspace,
                                    size_t workspace_bytes, void* cuda_stream);

/*
 * star_lse_merge — exact merge of per-split partials into global attention
 * [pith 2WVXFXZ2, minor comment on Algorithm 2 (corrected update
 * exp(s_h - s_global) * A_h); assumptions: online softmax aggregation gives
 * the exact global softmax]:
 *   m = max_h lse_h,  w_h = exp(lse_h - m),
 *   o = sum_h w_h o_h / sum_h w_h   -> o[B, T, Hq, D] bf16
 *   lse = m + log(sum_h w_h)        -> lse[B, Hq, T] fp32 (NULL to skip)
 * Splits whose lse is -inf carry weight 0. Inputs as star_phase2_partial
 * writes them.
 */
star_status star_lse_merge(const float* part_o, const float* part_lse, int nsplit, void* o,
                           float* lse, int B, int T, int Hq, int D, void* cuda_stream);

/*
 * star_lse_merge_ranks — star_lse_merge over partials gathered from several
 * ranks (the query host's aggregation step [pith 2WVXFXZ2, Referee summary]).
 * Every rank owns an equal slot of B * Hq * nsplit_stride * T * D floats of
 * part_o and B * Hq * nsplit_stride * T floats of part_lse (an all-gather of
 * equal-sized send buffers); rank r's slot begins with its nsplit_of_rank[r]
 * splits as star_phase2_partial_ext writes them, [B, Hq, nsplit_of_rank[r],
 * T, D] and [B, Hq, nsplit_of_rank[r], T]; the rest of the slot is ignored.
 * nsplit_of_rank is a host array, 0 <= nsplit_of_rank[r] <= nsplit_stride,
 * 1 <= nranks <= 64. Output and errors as star_lse_merge.
 */
star_status star_lse_merge_ranks(const float* part_o, const float* part_lse, int nranks,
                                 const int* nsplit_of_rank, int nsplit_stride, void* o, float* lse,
                                 int B, int T, int Hq, int D, void* cuda_stream);

/*
 * star_phase2_decode_static — star_phase2_partial for decode steps
 * (T * (Hq / Hkv) <= 16) without a workspace argument. The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory themselves, such as a plugin whose host application owns
 * every device allocation, or a serving loop that must never block in
 * cudaMalloc/cudaFree. Its scratch (the split counters and the per-chunk
 * partials) lives in a 16 MiB device array inside the library, which every
 * GPU that loads the library keeps until the process exits; the caller still
 * passes inputs and outputs, with the same meaning and layout as
 * star_phase2_partial.
 *   - The array's address is looked up once per device on the first call made
 *     with that device current; make that first call before any stream
 *     capture.
 *   - All calls on a device share the array, which keeps the previous call's
 *     contents: each call clears the split counters and rewrites the partials
 *     before reading them; device errors are ORed into a status word that
 *     stays set until star_phase2_decode_static_status reads it. Calls whose
 *     work overlaps on the GPU race on the array: serialise them (one stream,
 *     or explicit ordering).
 *   - Sizes whose scratch cannot fit 16 MiB even with the largest chunk, or
 *     T * g > 16, return STAR_ERR_INVALID_ARG before anything is enqueued.
 *     Nothing is allocated.
 */
star_status star_phase2_decode_static(const void* q, const void* k, const void* v, int T,
                                      void* k_cache, void* v_cache, int Lcap, int L,
                                      int block_len, int tail_len, float* part_o,
                                      float* part_lse, int* nsplit_out, int B, int Hq, int Hkv,
                                      int D, double theta, void* cuda_stream);

/*
 * star_phase2_decode_static_status — the device-error read-back of
 * star_phase2_decode_static, which has no workspace for star_device_status
 * to read. The pages have no counterpart. Synchronises `cuda_stream`, reads
 * the status word kept at the start of the current device's static array
 * (device errors of every star_phase2_decode_static call since the last
 * read are ORed into it: a bounded wait that gave up, an index outside its
 * buffer) and clears it. Returns STAR_OK, STAR_ERR_DEVICE_TIMEOUT or
 * STAR_ERR_DEVICE_BOUNDS (message in star_last_error), or STAR_ERR_CUDA.
 * After a device error the outputs of the calls since the last read are not
 * valid. Allocates nothing; the first call on a device looks up the array's
 * address like star_phase2_decode_static does.
 */
star_status star_phase2_decode_static_status(void* cuda_stream);

/*
 * Layers around Star attention in a decoder stack. Star Attention replaces
 * only attention and needs no retraining [pith 2WVXFXZ2, the paper's
 * abstract]; in a stack every layer encodes its own anchor, whose hidden
 * state is block 1's at that layer because the anchor is a causal prefix of
 * every augmented block [pith 2WVXFXZ2, "What carries the argument"]. These
 * two calls supply the row-wise parts of an attention block:
 *
 * star_rmsnorm — y[r, :] = x[r, :] / sqrt(mean(x[r, :]^2) + eps) * gamma,
 *   x, y bf16 [rows, dm] (row-major, may alias), gamma bf16 [dm]; fp32
 *   arithmetic, one rounding to bf16. dm a multiple of 8, pointers 16-byte
 *   aligned. STAR_ERR_INVALID_ARG otherwise; STAR_ERR_CUDA if the launch fails.
 *
 * star_linear — y[M, N] = x[M, K] * w[N, K]^T (accumulate = 0), or
 *   y = bf16(y + bf16(x * w^T)) (accumulate = 1: the stored projection, then
 *   the residual add), bf16 row-major operands, fp32 accumulation. It runs in
 *   the library's own tcgen05 GEMM (128 x 256 tiles, TMA-fed, persistent).
 *   N and K multiples of 8, x/w/y 16-byte aligned. workspace (caller-owned,
 *   256-byte aligned, >= 256 bytes, zero-filled once) holds the status word a
 *   bounded wait writes on a time-out (star_device_status reads it).
 *   STAR_ERR_INVALID_ARG for bad shapes or pointers, STAR_ERR_UNSUPPORTED off
 *   sm_100, STAR_ERR_CUDA for a failed launch.
 */
star_status star_rmsnorm(const void* x, const void* gamma, void* y, int rows, int dm, float eps,
                         void* cuda_stream);
star_status star_linear(const void* x, const void* w, void* y, int M, int N, int K, int accumulate,
                        void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * star_linear_rope — a Q/K/V projection whose output goes straight to where
 * Star attention reads it [pith 2WVXFXZ2, "What carries the argument": keys
 * keep their original position IDs; pith 2607.20457: original global
 * positions preserve RoPE distances]:
 *   p = bf16(x[M, K] * w[N, K]^T), rows m = b * seq_len + t (token t of
 *   sequence b), N = H * head_dim columns (H heads);
 *   rotate = 1: every head is rotated as star_rope does (rotate-half, base
 *   theta, position pos0 + t), from the bf16 values p, correctly rounded, so
 *   the bits equal star_linear followed by star_rope;
 *   cache_rows = 0: y is row-major [M, N] (token-major [B, seq_len, H, D]);
 *   cache_rows > 0: y is a head-major KV cache [B, H, cache_rows, head_dim]
 *   and token t of sequence b lands in row t (rows >= seq_len untouched).
 * A Phase-1 layer projects Q with rotate = 1, cache_rows = 0, K with
 * rotate = 1 into its k_cache and V with rotate = 0 into its v_cache, then
 * calls star_phase1_encode_rotated: no separate RoPE pass.
 * head_dim 64 or 128; N a multiple of head_dim; M a multiple of seq_len;
 * cache_rows 0 or >= seq_len; at least one of rotate and a cache layout.
 * workspace: >= star_linear_rope_workspace_bytes(seq_len, head_dim, rotate)
 * bytes, 256-byte aligned, zero-filled once: the status word, then (rotate)
 * the call's fp32 cos/sin table of its seq_len positions, built by a small
 * kernel the call launches before the GEMM. Operands and errors as
 * star_linear.
 */
size_t star_linear_rope_workspace_bytes(int seq_len, int head_dim, int rotate);

/*
 * star_linear_kv_cache — a layer's K and V projections as one GEMM, written
 * straight into its KV cache: w_kv[2N, K] holds the K projection's N rows
 * and then the V projection's N rows (N = Hkv * head_dim). With
 * p = bf16(x[M, K] * w_kv^T): columns [0, N) are the keys, rotated as
 * star_linear_rope rotates them (position pos0 + t), into k_cache; columns
 * [N, 2N) are the values, unrotated, into v_cache; both caches head-major
 * [M / seq_len, Hkv, cache_rows, head_dim], token t of sequence b in row t.
 * The bits equal star_linear_rope(K, rotate = 1) and star_linear_rope(V,
 * rotate = 0) on the two halves; one launch fills the GPU better than two
 * narrow ones. cache_rows >= seq_len; workspace as star_linear_rope with
 * rotate = 1. Errors as star_linear_rope.
 */
star_status star_linear_kv_cache(const void* x, const void* w_kv, void* k_cache, void* v_cache,
                                 int M, int N, int K, int head_dim, int seq_len, int64_t pos0,
                                 double theta, int cache_rows, void* workspace,
                                 size_t workspace_bytes, void* cuda_stream);
star_status star_linear_rope(const void* x, const void* w, void* y, int M, int N, int K,
                             int head_dim, int rotate, int seq_len, int64_t pos0, double theta,
                             int cache_rows, void* workspace, size_t workspace_bytes,
                             void* cuda_stream);

/*
 * star_device_status — synchronises `cuda_stream`, then reads the status
 * bits at the start of `workspace` (a workspace passed to any call; the bits
 * are sticky since the last read) and clears them. After a device error it
 * also clears the decode counters (the header size the last decode call
 * recorded in the status block), since an aborted call may leave them
 * non-zero. Returns STAR_OK, STAR_ERR_DEVICE_TIMEOUT or STAR_ERR_DEVICE_BOUNDS
 * (message in star_last_error), or STAR_ERR_CUDA.
 */
star_status star_device_status(void* workspace, void* cuda_stream);

/*
 * star_debug_wait_probe — checks the kernels' bounded waits and the status
 * read-back: one CTA waits, through the same bounded wait the attention and
 * decode kernels use, on a barrier nothing arrives on; after `seconds`
 * (0 < seconds <= 2) the wait gives up and records a time-out in the status
 * word at the start of `workspace` (>= 256 bytes, cleared first). A following
 * star_device_status returns STAR_ERR_DEVICE_TIMEOUT; nothing faults and the
 * context stays usable.
 */
star_status star_debug_wait_probe(void* workspace, double seconds, void* cuda_stream);

/*
 * star_debug_index — evaluates the kernels' index math on the device for
 * every context row r in [0, L): blk[r] = block id, pos[r] = position ID,
 * kv_ranges[4r..4r+3] = {anchor_lo, anchor_hi, own_lo, own_hi} (half-open;
 * block 0 reports an empty anchor range [0, 0)). Device int32 outputs.
 */
star_status star_debug_index(int L, int block_len, int anchor_len, int32_t* blk, int32_t* pos,
                             int32_t* kv_ranges, void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* STAR_H_ */
