/*
 * pagedkv.h -- C ABI of the B200 (sm_100a) paged-KV decode attention library
 * (libpagedkv.so).
 *
 * Operations and the passages that define them (web pages, by title/section):
 *   [VKV]  ybb.press "LLM 推理 KV Cache 内存管理深度工程实践：从 PageAttention 到推测解码":
 *          §2.1 BlockTable (block table, ceil block count, append_slot),
 *          §2.2 paged_attention_forward(query, paged_kv_cache, block_table,
 *          context_len, scale), §6.1 INT8/FP8 KV cache (quantize_kv_cache),
 *          §6.2 GQA (every G query heads share one KV head).
 *   [KVP]  t6page.pages.dev "KV cache": "PagedAttention 的算子" (K/V looked up
 *          through the block table, softmax taken over all blocks together).
 *   [KVL]  blog.hotdry.top "KV缓存内存布局优化": "PagedEviction 块级驱逐机制"
 *          (token importance S = ||V||_2 / ||K||_2, decode-phase eviction of the
 *          complete block with the lowest mean importance).
 *   [NANO] blog.hotdry.top nano-vLLM KV cache: the [2, L, blocks, bs, n_kv, d]
 *          tensor, reached here through per-layer K and V base pointers.
 *
 * Conventions shared by every entry point
 *   - All data pointers are DEVICE pointers owned by the caller; the library
 *     allocates nothing and keeps no state between calls except what the
 *     caller passes in (the decode workspace, the chunked-prefill workspace)
 *     and the one file-scope scratch array of pa_decode_static_scratch.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and returns after enqueueing.
 *   - Return value: PA_OK (0) when the work was enqueued; a negative PA_ERR_*
 *     code when an argument is invalid, in which case nothing is launched.
 *     Every call checks its arguments before any CUDA call (its "Host errors"
 *     line lists them); after that, PA_ERR_DEVICE when the current device is
 *     not an sm_100 GPU and PA_ERR_CUDA when a runtime call or launch fails.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Physical KV pool of one layer: [N blocks][bs slots][Hkv heads][d],
 *     element (blk, slot, h, e) at blk*block_stride + (slot*Hkv + h)*d + e,
 *     with block_stride >= bs*Hkv*d elements ([VKV] §2.2 shape
 *     [num_gpu_blocks, block_size, num_kv_heads, head_dim]).
 *   - Block table: int32 [B][MB] (MB = max blocks per sequence); entry j of row
 *     b is the physical block of logical block j.  Only entries below
 *     ceil(len_b / bs) are read.
 *   - Device-detected faults never trap: the kernel ORs a PA_DEV_* bit into
 *     *err_flag (a caller-zeroed device int32, required) and skips the
 *     offending block or sequence.
 *   - Supported sizes: d in {64, 128}; Hq % Hkv == 0 with G = Hq/Hkv <= 16;
 *     bs >= 1 (bs a multiple of 16 selects the staged tensor-core decode);
 *     pool/base pointers 16-byte aligned and block_stride*elt a multiple of 16;
 *     B <= 65535 and Hkv <= 65535 (grid limits), N <= 2^31 - 1 and
 *     MB*bs <= 2^31 - 1 (token positions are int32).  Outside these: PA_ERR_SHAPE.
 *   - Offsets into a pool are formed in 64 bits: N * block_stride may exceed
 *     2^31 elements (a pool of tens of GB is one pool).
 *   - pa_decode, pa_decode_int8, pa_decode_fp8, pa_decode_prepare with the
 *     planned calls, and pa_prefill_attention only enqueue kernels (no host
 *     synchronisation, copy or allocation), so a caller can capture them in a
 *     CUDA graph and replay it with new contents in the same buffers.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- host status codes ---------------------------------------------------- */
#define PA_OK             0
#define PA_ERR_NULL      -1  /* a required pointer is NULL                          */
#define PA_ERR_SHAPE     -2  /* unsupported or inconsistent sizes                   */
#define PA_ERR_ALIGN     -3  /* pointer or stride not 16-byte aligned               */
#define PA_ERR_WORKSPACE -4  /* workspace missing or smaller than required          */
#define PA_ERR_CUDA      -5  /* a CUDA runtime call or kernel launch failed          */
#define PA_ERR_DEVICE    -6  /* current device is not an sm_100 GPU                  */

/* ---- device error-flag bits (ORed into *err_flag) ------------------------- */
#define PA_DEV_BAD_BLOCK  1  /* a needed block-table entry was outside [0, N)       */
#define PA_DEV_BAD_LEN    2  /* a context length / position outside [0, MB*bs]     */
#define PA_DEV_TIMEOUT    4  /* a bounded pipeline wait gave up (kernel returned)   */
#define PA_DEV_BAD_EVICT  8  /* an eviction index that is not a full block          */
#define PA_DEV_BAD_PLAN  16  /* the workspace holds no plan for these sizes         */

/* Human-readable text of a PA_* status code (static storage). */
const char *pa_status_string(int code);

/* Library version string (static storage). */
const char *pa_version(void);

/* ============================================================================
 * a1. KV append  ([VKV] §2.1 append_slot)
 *
 * Writes n_new tokens per sequence into the paged pools.  Token i of sequence b
 * (i < n_new) has position p = positions[b] + i and lands in
 *     slot = block_tables[b][p / bs] * bs + p % bs,
 * i.e. physical block block_tables[b][p / bs], offset p % bs, for every kv head.
 * n_new = 1 is the decode-step append; n_new > 1 writes a prompt (prefill).
 * The caller's allocator must already have placed every needed block in the
 * table (the append allocates nothing).
 *   k_new, v_new : [B][n_new][Hkv][d] bf16, contiguous.
 *   k_cache, v_cache : one layer's pools (see conventions), written.
 *   slot_out     : optional [B][n_new] int64, receives the slots (NULL = skip).
 * Device errors: p outside [0, MB*bs) -> PA_DEV_BAD_LEN; table entry outside
 * [0, N) -> PA_DEV_BAD_BLOCK; that token is skipped.
 * Host errors: B = 0 or n_new = 0 -> PA_OK (nothing to do); a NULL k_new, v_new,
 * pool, table, positions or err_flag -> PA_ERR_NULL; n_new < 0 or sizes outside
 * the supported ranges -> PA_ERR_SHAPE; k_new, v_new or a pool not 16-byte
 * aligned, or block_stride*2 not a multiple of 16 -> PA_ERR_ALIGN.
 * ==========================================================================*/
int pa_append_kv(const uint16_t *k_new, const uint16_t *v_new,
                 uint16_t *k_cache, uint16_t *v_cache, int64_t block_stride,
                 const int32_t *block_tables, int max_blocks_per_seq,
                 const int32_t *positions, int B, int n_new, int Hkv, int d, int bs,
                 int64_t num_blocks, int64_t *slot_out, int32_t *err_flag, void *stream);

/* ============================================================================
 * a2 + a3. Paged decode attention  ([VKV] §2.2; [KVP] operator; [VKV] §6.2)
 *
 * For every sequence b and query head i, with G = Hq / Hkv and kv head
 * h = i / G (contiguous GQA groups):
 *     out[b][i] = sum_t softmax_t(scale * q[b][i] . K[b, t, h]) V[b, t, h]
 * over the tokens t < ctx_lens[b] read through the block table, the softmax
 * being taken over the whole context.  Computed with an online softmax in fp32
 * over a split-KV partition of the context, then a log-sum-exp merge of the
 * partitions; the result is rounded to bf16 (nearest-even).  ctx_lens[b] == 0
 * gives a zero row.
 *   out : [B][Hq][d] bf16, written.          q : [B][Hq][d] bf16.
 *   ctx_lens : [B] int32 in [0, MB*bs] (the appended token included).
 *   num_splits : maximum partitions per sequence; 0 = choose automatically.
 *   workspace  : device scratch of at least pa_decode_workspace_bytes(...)
 *                bytes for the same sizes and num_splits (may be NULL when that
 *                is 0).  Its contents are scratch; calls sharing one workspace
 *                must be ordered on one stream.
 * Device errors: ctx_lens[b] outside [0, MB*bs] -> PA_DEV_BAD_LEN (row zeroed);
 * a needed table entry outside [0, N) -> PA_DEV_BAD_BLOCK (block skipped).
 * Host errors: B = 0 -> PA_OK; a NULL out, q, pool, table, ctx_lens or err_flag
 * -> PA_ERR_NULL; Hq not a positive multiple of Hkv, G > 16, a NaN scale or sizes
 * outside the supported ranges -> PA_ERR_SHAPE; out, q, a pool or the workspace not
 * 16-byte aligned, or block_stride*2 not a multiple of 16 -> PA_ERR_ALIGN; the
 * workspace NULL or smaller than pa_decode_workspace_bytes when that is > 0 ->
 * PA_ERR_WORKSPACE.  pa_decode_workspace_bytes returns 0 for invalid sizes;
 * pa_decode_plan returns PA_ERR_NULL for a NULL num_splits_out or
 * chunk_tokens_out and PA_ERR_SHAPE for invalid sizes.
 * ==========================================================================*/
size_t pa_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int bs,
                                 int max_blocks_per_seq, int num_splits);

/* The partition pa_decode chooses for these sizes (no counterpart in the pages:
 * the split-KV partition exists only in this implementation).  *num_splits_out
 * receives the maximum number of partitions of one sequence, *chunk_tokens_out
 * the tokens per partition (for the staged kernel: the minimum; it sizes the
 * partitions from the actual lengths on the device), *launches_out (nullable)
 * the kernels one pa_decode call launches, *staged_out (nullable) 1 when the
 * staged tensor-core kernel runs (a plan kernel, the decode kernel, then a
 * merge kernel when a sequence has several partial results), 0 for the
 * general-shape kernel (decode, then a merge kernel when partitions > 1).
 * Returns PA_OK or a PA_ERR_* code. */
int pa_decode_plan(int B, int Hq, int Hkv, int d, int bs, int max_blocks_per_seq,
                   int num_splits, int *num_splits_out, int *chunk_tokens_out,
                   int *launches_out, int *staged_out);

int pa_decode(uint16_t *out, const uint16_t *q,
              const uint16_t *k_cache, const uint16_t *v_cache, int64_t block_stride,
              const int32_t *block_tables, int max_blocks_per_seq, const int32_t *ctx_lens,
              int B, int Hq, int Hkv, int d, int bs, int64_t num_blocks, float scale,
              int num_splits, void *workspace, size_t workspace_bytes,
              int32_t *err_flag, void *stream);

/* ============================================================================
 * a4. PagedEviction token importance  ([KVL] "PagedEviction 块级驱逐机制")
 *
 *   scores[b][t][h] = ||V[b, t, h, :]||_2 / ||K[b, t, h, :]||_2   (fp32)
 * for t < ctx_lens[b] and every kv head h, on the stored bf16 values.  When
 * ||K|| == 0 the score is +inf if ||V|| > 0, else 0.  Entries with
 * t >= ctx_lens[b] are not written.
 *   scores : [B][MB*bs][Hkv] fp32.
 * Device errors: ctx_lens[b] outside [0, MB*bs] -> PA_DEV_BAD_LEN (sequence
 * skipped); a table entry outside [0, N) -> PA_DEV_BAD_BLOCK (block skipped).
 * Host errors: B = 0 -> PA_OK; a NULL scores, pool, table, ctx_lens or err_flag ->
 * PA_ERR_NULL; sizes outside the supported ranges -> PA_ERR_SHAPE; a pool not
 * 16-byte aligned or block_stride*2 not a multiple of 16 -> PA_ERR_ALIGN.
 * ==========================================================================*/
int pe_score_tokens(float *scores, const uint16_t *k_cache, const uint16_t *v_cache,
                    int64_t block_stride, const int32_t *block_tables, int max_blocks_per_seq,
                    const int32_t *ctx_lens, int B, int Hkv, int d, int bs,
                    int64_t num_blocks, int32_t *err_flag, void *stream);

/* ============================================================================
 * a5. PagedEviction block selection  ([KVL] "PagedEviction 块级驱逐机制")
 *
 * For each sequence, over its FULL logical blocks j < floor(ctx_lens[b] / bs):
 *   mean_j = (1 / (bs*Hkv)) * sum_{t in block j, h} scores[b][t][h]
 * accumulated in fp64 (exact for the fp32 scores of one block), and
 *   evict[b] = argmin_j mean_j  (lowest j on ties), or -1 if no block is full.
 * The caller maps evict[b] to the physical block block_tables[b][evict[b]],
 * drops it from the table and frees it (host bookkeeping, not done here).
 *   evict       : [B] int32, written.
 *   block_means : optional [B][MB] fp32 (fp64 mean rounded to nearest); NaN for
 *                 non-candidate blocks.  NULL = skip.
 *   scores      : [B][MB*bs][Hkv] fp32 as written by pe_score_tokens.
 * A length outside [0, MB*bs] counts as 0 (no full block: -1); there is no
 * error flag.  Host errors: B = 0 -> PA_OK; a NULL evict, scores or ctx_lens ->
 * PA_ERR_NULL; B < 0, MB < 1, Hkv < 1 or bs < 1 -> PA_ERR_SHAPE.
 * ==========================================================================*/
int pe_select_evict_block(int32_t *evict, float *block_means, const float *scores,
                          const int32_t *ctx_lens, int B, int max_blocks_per_seq, int Hkv,
                          int bs, void *stream);

/* ============================================================================
 * a6. INT8 KV append  ([VKV] §6.1 quantize_kv_cache; [VKV] §2.1 append_slot)
 *
 * As pa_append_kv, but every (token, kv head) row x[0..d) is quantised first:
 *   s = max_e |x_e| / 127            (one IEEE fp32 division)
 *   code_e = round_half_even(x_e / s) (IEEE fp32 division), int8 in [-127, 127]
 *   s == 0  ->  all codes 0.
 *   kq_cache, vq_cache : int8 pools [N][bs][Hkv][d] (block_stride elements).
 *   k_scale, v_scale   : fp32 scale pools [N][bs][Hkv] (block stride bs*Hkv).
 * Host errors: as pa_append_kv, plus a NULL scale pool -> PA_ERR_NULL, and scale
 * pools not 16-byte aligned or block_stride not a multiple of 16 -> PA_ERR_ALIGN.
 * ==========================================================================*/
int pa_append_kv_int8(const uint16_t *k_new, const uint16_t *v_new,
                      int8_t *kq_cache, int8_t *vq_cache, float *k_scale, float *v_scale,
                      int64_t block_stride, const int32_t *block_tables, int max_blocks_per_seq,
                      const int32_t *positions, int B, int n_new, int Hkv, int d, int bs,
                      int64_t num_blocks, int64_t *slot_out, int32_t *err_flag, void *stream);

/* ============================================================================
 * a7. INT8 paged decode  ([VKV] §6.1 dequantisation; otherwise as pa_decode)
 *
 * pa_decode with K[t, h, e] = k_scale[t, h] * kq[t, h, e] and likewise V,
 * dequantised in registers (the K scale multiplies the dot product, the V
 * scale multiplies the softmax weight).  Same workspace rule as pa_decode.
 * k_scale, v_scale: fp32 [N][bs][Hkv], 16-byte aligned (PA_ERR_ALIGN otherwise).
 * The query stays bf16 (the page quantises the cache only).  With d = 128 and
 * bs a multiple of 16 the dot products q.kq run on int8 tensor cores: each
 * query row is scaled by a power of two, rounded to integers of magnitude at
 * most 8355711 (23 bits) and split exactly into three int8 parts, so the one
 * approximation is that rounding, below 2^-23 of the row's largest |q| per
 * element (rows whose largest |q| is at least 2^-104).  Other shapes compute
 * in fp32 from the bf16 query.  Any finite bf16 query whose logits are finite
 * in fp32 is valid.
 * Host errors: as pa_decode, plus a NULL scale pool -> PA_ERR_NULL and
 * block_stride not a multiple of 16 -> PA_ERR_ALIGN.
 * ==========================================================================*/
int pa_decode_int8(uint16_t *out, const uint16_t *q,
                   const int8_t *kq_cache, const int8_t *vq_cache,
                   const float *k_scale, const float *v_scale, int64_t block_stride,
                   const int32_t *block_tables, int max_blocks_per_seq, const int32_t *ctx_lens,
                   int B, int Hq, int Hkv, int d, int bs, int64_t num_blocks, float scale,
                   int num_splits, void *workspace, size_t workspace_bytes,
                   int32_t *err_flag, void *stream);

/* ============================================================================
 * FP8 (e4m3) KV  ([VKV] §6.1: the FP8 branch of quantize_kv_cache casts the
 * KV tensor to float8_e4m3fn, without a scale)
 *
 * pa_append_kv_fp8: pa_append_kv storing each element as an e4m3 code (1 sign,
 * 4 exponent bits with bias 7, 3 mantissa bits): round to nearest, ties to
 * even; finite values beyond +-448 saturate to +-448 (reading: the page's cast
 * does not say; saturation keeps the cache finite); NaN stays NaN.
 *   k8_cache, v8_cache : uint8 pools [N][bs][Hkv][d] (block_stride elements).
 * pa_decode_fp8: pa_decode over e4m3 pools; every code is widened exactly (each
 * e4m3 value is an fp16 value) in registers.  Same workspace rule as pa_decode.
 * With d = 128 and bs a multiple of 16 the products run on fp16 tensor cores:
 * each bf16 query row is first scaled by a power of two that puts its largest
 * |q| in [2^14, 2^15), so no query overflows fp16 (|q| > 65504 included) and
 * every element down to 2^-32 of the row's largest converts exactly; the scale
 * is taken back on the logit.  Any finite bf16 query whose logits are finite
 * in fp32 is valid.
 * Host errors: as pa_append_kv and pa_decode, with block_stride (one-byte
 * elements) a multiple of 16 -> else PA_ERR_ALIGN.
 * ==========================================================================*/
int pa_append_kv_fp8(const uint16_t *k_new, const uint16_t *v_new,
                     uint8_t *k8_cache, uint8_t *v8_cache, int64_t block_stride,
                     const int32_t *block_tables, int max_blocks_per_seq,
                     const int32_t *positions, int B, int n_new, int Hkv, int d, int bs,
                     int64_t num_blocks, int64_t *slot_out, int32_t *err_flag, void *stream);

int pa_decode_fp8(uint16_t *out, const uint16_t *q,
                  const uint8_t *k8_cache, const uint8_t *v8_cache, int64_t block_stride,
                  const int32_t *block_tables, int max_blocks_per_seq, const int32_t *ctx_lens,
                  int B, int Hq, int Hkv, int d, int bs, int64_t num_blocks, float scale,
                  int num_splits, void *workspace, size_t workspace_bytes,
                  int32_t *err_flag, void *stream);

/* ============================================================================
 * One partition plan for several decode calls (no counterpart in the pages:
 * the split-KV partition exists only in this implementation).
 *
 * The staged decode's plan (every sequence's partitions, listed longest first)
 * depends only on ctx_lens and the sizes, which are the same for every layer of
 * a decode step.  pa_decode_prepare writes that plan into a workspace (one plan
 * launch); pa_decode_planned, pa_decode_int8_planned and pa_decode_fp8_planned
 * are pa_decode, pa_decode_int8 and pa_decode_fp8 taking the plan from the
 * workspace instead of making it, so each call launches one kernel fewer.  Their
 * arguments are those of the plain calls, and their results are bit for bit the
 * same, provided that
 *   - pa_decode_prepare ran on this workspace, ordered before the call on the
 *     same stream, with the same ctx_lens contents and the same B, Hq, Hkv, d,
 *     bs, max_blocks_per_seq and num_splits, and
 *   - no plain pa_decode* call and no other pa_decode_prepare used the workspace
 *     in between (a planned call leaves the plan ready for the next one).
 * One plan serves bf16, INT8 and FP8 calls of the same sizes.  The plan records
 * a signature of its sizes: a planned call of other sizes computes nothing,
 * raises PA_DEV_BAD_PLAN and leaves out untouched.  Changed ctx_lens contents are
 * not detected (the call then attends the ranges of the old lengths, reading
 * only table entries below max_blocks_per_seq): prepare again after a change.
 * Shapes served by the general-shape kernel keep no plan: pa_decode_prepare
 * launches nothing and the planned calls run as the plain ones.
 * Host errors: pa_decode_prepare: B = 0 -> PA_OK; a NULL ctx_lens or err_flag ->
 * PA_ERR_NULL; sizes outside the supported ranges -> PA_ERR_SHAPE; the workspace
 * NULL or smaller than pa_decode_workspace_bytes -> PA_ERR_WORKSPACE, not 16-byte
 * aligned -> PA_ERR_ALIGN.  The planned calls: as the plain ones.
 * ==========================================================================*/
int pa_decode_prepare(const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs,
                      int max_blocks_per_seq, int num_splits, void *workspace,
                      size_t workspace_bytes, int32_t *err_flag, void *stream);

int pa_decode_planned(uint16_t *out, const uint16_t *q,
                      const uint16_t *k_cache, const uint16_t *v_cache, int64_t block_stride,
                      const int32_t *block_tables, int max_blocks_per_seq,
                      const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs,
                      int64_t num_blocks, float scale, int num_splits, void *workspace,
                      size_t workspace_bytes, int32_t *err_flag, void *stream);

int pa_decode_int8_planned(uint16_t *out, const uint16_t *q,
                           const int8_t *kq_cache, const int8_t *vq_cache,
                           const float *k_scale, const float *v_scale, int64_t block_stride,
                           const int32_t *block_tables, int max_blocks_per_seq,
                           const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs,
                           int64_t num_blocks, float scale, int num_splits, void *workspace,
                           size_t workspace_bytes, int32_t *err_flag, void *stream);

int pa_decode_fp8_planned(uint16_t *out, const uint16_t *q,
                          const uint8_t *k8_cache, const uint8_t *v8_cache, int64_t block_stride,
                          const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs,
                          int64_t num_blocks, float scale, int num_splits, void *workspace,
                          size_t workspace_bytes, int32_t *err_flag, void *stream);

/* ============================================================================
 * Incremental PagedEviction scoring  ([KVL] "PagedEviction 块级驱逐机制": the
 * importance S = ||V||_2 / ||K||_2 needs only the token's own K and V, and in
 * the decode phase a block is chosen only when the newest block fills)
 *
 * pa_append_kv_scored: pa_append_kv that also writes each new (token, kv head)
 * score into score_pool at the token's slot.  score_pool is fp32
 * [N][bs][Hkv] (block stride bs*Hkv), paged exactly like the KV pool, so a
 * block's scores move, stay and are freed with its K/V.  The score is computed
 * from the bf16 values written, as pe_score_tokens would compute it from the
 * pool (same ||K|| == 0 rule).
 * pa_append_kv_int8_scored: the same for the INT8 append; the score is taken on
 * the dequantised row (scale * codes).
 * pe_select_evict_block_pooled: pe_select_evict_block reading the scores of
 * every full logical block j < floor(ctx_lens[b] / bs) from score_pool through
 * the block table (physical block block_tables[b][j]), summed in the same order
 * and precision, so it returns exactly what pe_select_evict_block returns on
 * the equal [B][MB*bs][Hkv] score array.  A needed table entry outside [0, N)
 * raises PA_DEV_BAD_BLOCK and that block is not a candidate.
 * Host errors: the appends as pa_append_kv / pa_append_kv_int8, plus a NULL
 * score_pool -> PA_ERR_NULL.  pe_select_evict_block_pooled: B = 0 -> PA_OK; a NULL
 * evict, score_pool, table, ctx_lens or err_flag -> PA_ERR_NULL; B outside
 * [0, 65535], MB < 1, Hkv < 1, bs < 1 or N < 1 -> PA_ERR_SHAPE.
 * ==========================================================================*/
int pa_append_kv_scored(const uint16_t *k_new, const uint16_t *v_new,
                        uint16_t *k_cache, uint16_t *v_cache, int64_t block_stride,
                        float *score_pool, const int32_t *block_tables, int max_blocks_per_seq,
                        const int32_t *positions, int B, int n_new, int Hkv, int d, int bs,
                        int64_t num_blocks, int64_t *slot_out, int32_t *err_flag, void *stream);

int pa_append_kv_int8_scored(const uint16_t *k_new, const uint16_t *v_new,
                             int8_t *kq_cache, int8_t *vq_cache, float *k_scale, float *v_scale,
                             float *score_pool, int64_t block_stride,
                             const int32_t *block_tables, int max_blocks_per_seq,
                             const int32_t *positions, int B, int n_new, int Hkv, int d, int bs,
                             int64_t num_blocks, int64_t *slot_out, int32_t *err_flag,
                             void *stream);

int pe_select_evict_block_pooled(int32_t *evict, float *block_means, const float *score_pool,
                                 const int32_t *block_tables, int max_blocks_per_seq,
                                 const int32_t *ctx_lens, int B, int Hkv, int bs,
                                 int64_t num_blocks, int32_t *err_flag, void *stream);

/* ============================================================================
 * Decode and pooled block selection in one call ([KVL] "PagedEviction 块级驱逐
 * 机制": in the decode phase the block to evict is chosen from the scores of
 * complete blocks; the choice does not depend on the attention output)
 *
 * pa_decode_select_pooled is pa_decode followed by pe_select_evict_block_pooled
 * on the same block_tables, ctx_lens, B, max_blocks_per_seq, Hkv, bs and
 * num_blocks; pa_decode_planned_select_pooled is the same with pa_decode_planned
 * (same plan rules).  out is what the decode call gives and evict / block_means
 * what the selection call gives, bit for bit.  The selection runs in B extra CTAs
 * at the front of the decode's merge launch, beside the decode kernel, so a decode
 * layer with incremental eviction is the scored append plus the decode's launches
 * (plan, decode, merge; no plan for the planned call).  Where the decode has no
 * merge launch (a single partition, or the general-shape kernel), or merges with
 * one CTA per row, the selection kernel is launched after it instead.  The score
 * pool, tables and lengths are only read; the selection's results do not depend
 * on the plan (a refused plan still gets them).  Only the bf16 decode has this form.
 * Host errors: those of either call; a NULL evict or score_pool -> PA_ERR_NULL
 * (block_means may be NULL).
 * ==========================================================================*/
int pa_decode_select_pooled(uint16_t *out, const uint16_t *q,
                            const uint16_t *k_cache, const uint16_t *v_cache,
                            int64_t block_stride, const int32_t *block_tables,
                            int max_blocks_per_seq, const int32_t *ctx_lens, int B, int Hq,
                            int Hkv, int d, int bs, int64_t num_blocks, float scale,
                            int num_splits, void *workspace, size_t workspace_bytes,
                            int32_t *evict, float *block_means, const float *score_pool,
                            int32_t *err_flag, void *stream);

int pa_decode_planned_select_pooled(uint16_t *out, const uint16_t *q,
                                    const uint16_t *k_cache, const uint16_t *v_cache,
                                    int64_t block_stride, const int32_t *block_tables,
                                    int max_blocks_per_seq, const int32_t *ctx_lens, int B,
                                    int Hq, int Hkv, int d, int bs, int64_t num_blocks,
                                    float scale, int num_splits, void *workspace,
                                    size_t workspace_bytes, int32_t *evict, float *block_means,
                                    const float *score_pool, int32_t *err_flag, void *stream);

/* ============================================================================
 * pa_decode without a caller-provided workspace (no counterpart in the pages;
 * it exists for callers, not for the method).
 *
 * Some callers cannot allocate device memory: a host runtime whose memory
 * manager owns every byte of the GPU and forbids raw allocations, a plain-C
 * caller that holds only device pointers handed to it, or a process that has
 * reserved its whole memory budget at start-up.  For them this entry point
 * computes what pa_decode computes, with the same arguments minus the
 * workspace, and takes its scratch from a fixed array that lives inside the
 * library: PA_STATIC_SCRATCH_BYTES (16 MiB) on every GPU that loads the library,
 * held until the process exits.  It allocates nothing.
 *   num_splits : as pa_decode when the scratch of that plan fits the array (then
 *                the call launches exactly what pa_decode launches, bit for bit
 *                the same result).  When num_splits = 0 and the automatic plan's
 *                scratch does not fit, the call takes the largest partition count
 *                whose scratch fits (so it may partition, and round, differently
 *                from pa_decode).  When the scratch needed for the given sizes
 *                and a non-zero num_splits exceeds the array, the call returns
 *                PA_ERR_WORKSPACE and launches nothing.
 *   Every call looks up the array's device address with the calling device
 *   current (a host-side lookup that allocates nothing and follows a reset
 *   context).  The first call on a device may load the library's device code:
 *   make it before any stream capture.
 *   All calls on a device share the one array: two calls whose kernels overlap
 *   on the GPU (different streams, or different host threads) race and give
 *   wrong results; order them on one stream.  Nothing in the array needs to
 *   start at zero: every call writes what it later reads.
 * Host errors: as pa_decode without the workspace ones, plus num_splits < 0 ->
 * PA_ERR_SHAPE and scratch that does not fit -> PA_ERR_WORKSPACE.
 * ==========================================================================*/
#define PA_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)

int pa_decode_static_scratch(uint16_t *out, const uint16_t *q,
                             const uint16_t *k_cache, const uint16_t *v_cache,
                             int64_t block_stride, const int32_t *block_tables,
                             int max_blocks_per_seq, const int32_t *ctx_lens, int B, int Hq,
                             int Hkv, int d, int bs, int64_t num_blocks, float scale,
                             int num_splits, int32_t *err_flag, void *stream);

/* ============================================================================
 * PagedEviction prefill stage  ([KVL] "PagedEviction 块级驱逐机制", two-stage
 * strategy: at prefill each token gets an importance and the lowest-scoring
 * tokens are evicted down to the cache budget; the survivors fill whole blocks).
 *
 * Prompts arrive contiguous and token-major: k, v [T][Hkv][d] bf16 (all B
 * prompts concatenated; cu_seqlens [B+1] int32 device array of offsets, prompt b
 * = tokens cu_seqlens[b] .. cu_seqlens[b+1]-1).  d in {64, 128, 256}; k, v and
 * the pools 16-byte aligned.
 *
 * pe_prefill_scores: scores[t] (fp32, [T]) = mean over the Hkv heads of
 *   ||V[t,h]||_2 / ||K[t,h]||_2 (fp32 sums of squares; ||K|| = 0 gives +inf when
 *   ||V|| > 0, else 0).  Reading: a token is kept or evicted for all heads at
 *   once (one slot holds them all), so its importance is the head mean.
 *
 * pe_prefill_select: per prompt, the source indices of the tokens that stay.
 *   The budget tokens that rank highest stay; ranking is by score (numeric
 *   order, NaN counted as -inf, -0 equal to +0), and on equal scores the
 *   earlier token is evicted first.  Kept tokens keep their prompt order.
 *   keep_idx [B][budget] int32: prompt-local index of the p-th kept token, -1
 *   after the last; kept_len [B] = min(prompt length, budget).  budget >= 1.
 *   A negative prompt length sets PA_DEV_BAD_LEN and keeps nothing.
 *
 * pe_prefill_pack: writes the p-th kept token of prompt b (p < kept_len[b]) at
 *   position p of sequence b, slot = block_tables[b][p/bs]*bs + p%bs (every kv
 *   head), so the compressed prompt fills ceil(kept/bs) blocks densely.  The
 *   caller's allocator has placed those blocks in the table.  An index outside
 *   the prompt or p/bs >= MB sets PA_DEV_BAD_LEN; a block id outside [0, N)
 *   sets PA_DEV_BAD_BLOCK; the token is skipped.
 *
 * pe_prefill_compress: pe_prefill_scores, pe_prefill_select and
 *   pe_prefill_pack in one call (three launches on `stream`); scores,
 *   keep_idx and kept_len are outputs the caller may read afterwards.
 *
 * Host errors: pe_prefill_scores: T = 0 -> PA_OK; a NULL scores, k or v ->
 *   PA_ERR_NULL; T < 0, Hkv outside [1, 65535] or d not in {64, 128, 256} ->
 *   PA_ERR_SHAPE; k or v not 16-byte aligned -> PA_ERR_ALIGN.
 *   pe_prefill_select: B = 0 -> PA_OK; a NULL argument -> PA_ERR_NULL; B < 0 or
 *   budget < 1 -> PA_ERR_SHAPE.
 *   pe_prefill_pack: B = 0 -> PA_OK; a NULL pool, table, k, v, cu_seqlens,
 *   keep_idx, kept_len or err_flag -> PA_ERR_NULL; Hkv or d as for
 *   pe_prefill_scores, B < 0, budget < 1, bs < 1, MB < 1, N < 1 or
 *   block_stride < bs*Hkv*d -> PA_ERR_SHAPE; pools, k or v not 16-byte
 *   aligned, or block_stride*2 not a multiple of 16 -> PA_ERR_ALIGN.
 *   pe_prefill_compress: the union of the three, checked before the first
 *   launch (a NULL scores with T > 0 -> PA_ERR_NULL).
 * ==========================================================================*/
int pe_prefill_scores(float *scores, const uint16_t *k, const uint16_t *v, int64_t T, int Hkv,
                      int d, void *stream);

int pe_prefill_select(int32_t *keep_idx, int32_t *kept_len, const float *scores,
                      const int32_t *cu_seqlens, int B, int budget, int32_t *err_flag,
                      void *stream);

int pe_prefill_pack(uint16_t *k_cache, uint16_t *v_cache, int64_t block_stride,
                    const int32_t *block_tables, int max_blocks_per_seq, const uint16_t *k,
                    const uint16_t *v, const int32_t *cu_seqlens, const int32_t *keep_idx,
                    const int32_t *kept_len, int B, int budget, int Hkv, int d, int bs,
                    int64_t num_blocks, int32_t *err_flag, void *stream);

int pe_prefill_compress(uint16_t *k_cache, uint16_t *v_cache, int64_t block_stride,
                        const int32_t *block_tables, int max_blocks_per_seq, const uint16_t *k,
                        const uint16_t *v, const int32_t *cu_seqlens, int64_t T, int B,
                        int budget, int Hkv, int d, int bs, int64_t num_blocks, float *scores,
                        int32_t *keep_idx, int32_t *kept_len, int32_t *err_flag, void *stream);

/* ============================================================================
 * Block-table compaction after a decode-phase eviction  ([KVL] "PagedEviction
 * 块级驱逐机制": eviction removes whole blocks, never part of one).
 *
 * For every sequence b with evict[b] = j >= 0 (the logical index that
 * pe_select_evict_block returned): entries j+1 .. ceil(len_b/bs)-1 of
 * block_tables[b] move down by one, the last used entry becomes -1,
 * ctx_lens[b] drops by bs, and freed[b] (nullable [B]) receives the physical id
 * that left the table (the caller's allocator takes it back).  evict[b] < 0
 * leaves sequence b alone (freed[b] = -1).  Physical blocks do not move, so the
 * cached rows and a score pool stay valid.  j not a full block (j >= len/bs)
 * sets PA_DEV_BAD_EVICT, a length outside [0, MB*bs] PA_DEV_BAD_LEN; the
 * sequence is left unchanged.  block_tables and ctx_lens are updated in place.
 * Host errors: B = 0 -> PA_OK; a NULL block_tables, ctx_lens, evict or err_flag
 * -> PA_ERR_NULL; B < 0, MB < 1, bs < 1 or MB*bs > 2^31 - 1 -> PA_ERR_SHAPE.
 * ==========================================================================*/
int pe_evict_compact(int32_t *block_tables, int max_blocks_per_seq, int32_t *ctx_lens,
                     int32_t *freed, const int32_t *evict, int B, int bs, int32_t *err_flag,
                     void *stream);

/* ============================================================================
 * Threshold eviction policy  (blog.hotdry.top nano-vLLM KV cache page, section
 * "工程落地：参数配置与监控要点": eviction_ratio = 0.2 starts eviction once the
 * cache is more than 80 % used; blocks below importance_threshold go first).
 *
 * pe_select_evict_threshold: the trigger is evaluated on the host, in fp64, as
 *   used_blocks > (1 - eviction_ratio) * total_blocks (the caller's allocator
 *   counts).  Triggered: for each sequence every full block whose mean
 *   importance (as in pe_select_evict_block) is below importance_threshold is
 *   marked; a sequence with no such block marks its single lowest-mean full
 *   block (ties to the lowest index); no full block marks nothing.  Not
 *   triggered: nothing is marked.  Reading: the page gives the two parameters
 *   and their intent, not how many blocks go; this is the plainest rule that
 *   honours both and reduces to the decode-phase rule when nothing is below
 *   the threshold.
 *   mask [B][MB] uint8 (1 = evict), count [B] int32 (marked blocks),
 *   block_means (nullable) [B][MB] float, NaN for non-candidates.
 *   eviction_ratio in [0, 1]; importance_threshold not NaN.
 *
 * pe_evict_compact_mask: pe_evict_compact for any number of marked full blocks
 *   per sequence: marked full blocks leave the table, the other entries keep
 *   their order and close up, ctx_lens[b] drops by bs per removed block, and
 *   freed (nullable [B][MB]) lists the removed physical ids in logical order,
 *   -1 after the last.  A mark on the partial last block sets
 *   PA_DEV_BAD_EVICT and is ignored; marks at j >= ceil(len/bs) are not read.
 *
 * Host errors: pe_select_evict_threshold: B = 0 -> PA_OK; a NULL mask, count,
 *   scores or ctx_lens -> PA_ERR_NULL; B < 0, MB < 1, Hkv < 1, bs < 1, eviction_ratio
 *   outside [0, 1] (or NaN), a NaN importance_threshold or a negative block
 *   count -> PA_ERR_SHAPE.  pe_evict_compact_mask: as pe_evict_compact, with mask
 *   in place of evict.
 * ==========================================================================*/
int pe_select_evict_threshold(uint8_t *mask, int32_t *count, float *block_means,
                              const float *scores, const int32_t *ctx_lens, int B,
                              int max_blocks_per_seq, int Hkv, int bs, int64_t used_blocks,
                              int64_t total_blocks, double eviction_ratio,
                              double importance_threshold, void *stream);

int pe_evict_compact_mask(int32_t *block_tables, int max_blocks_per_seq, int32_t *ctx_lens,
                          int32_t *freed, const uint8_t *mask, int B, int bs, int32_t *err_flag,
                          void *stream);

/* ============================================================================
 * Multi-query paged attention for a chunked prefill  (t6page.pages.dev "KV
 * cache", "Chunked prefill：让 prefill 不阻塞 decode": a long prompt is prefilled
 * in chunks, 512 tokens each, batched with the running decodes; the operator is
 * the paged attention of "PagedAttention 的算子" / [VKV] §2.2 with several query
 * tokens per sequence).
 *
 * Sequence b has q_len_b = cu_q[b+1] - cu_q[b] query tokens, rows cu_q[b] ..
 * cu_q[b+1]-1 of q and out ([Tq][Hq][d] bf16, Tq = cu_q[B]).  Its chunk's K/V
 * rows were appended before the call (pa_append_kv with n_new = q_len_b), so
 * the queries are the last q_len_b of its ctx_lens[b] cached tokens: query i
 * sits at position p = ctx_lens[b] - q_len_b + i and attends exactly the tokens
 * t <= p (causal), softmax over all of them, GQA groups as in pa_decode.
 * q_len_b = 1 is a decode step (pa_decode is the faster call for those).
 * max_q_len >= every q_len_b (sizes the grid).  d in {64, 128}; G = Hq/Hkv in
 * {1, 2, 4, 8, 16}.  A sequence with q_len_b > ctx_lens[b] or a length outside
 * [0, MB*bs] gets zero output rows and sets PA_DEV_BAD_LEN; a block id outside
 * [0, N) sets PA_DEV_BAD_BLOCK and reads as zeros.
 *   workspace (nullable) : device scratch of at least
 *     pa_prefill_attention_workspace_bytes(...) bytes for the same sizes.  With it
 *     (d = 128, block size a multiple of 16) the work is balanced over the SMs: with
 *     n query tiles of 256 rows and P SMs, floor(n / P) P tiles run whole, one CTA
 *     each; the K/V ranges of the others are laid end to end and cut into one equal
 *     range per SM, and a range cut inside a tile leaves fp32 partial results (O,
 *     max, sum) in the workspace, merged with the log-sum-exp rule by the part that
 *     finishes last.  It pays off when the tiles are fewer than the SMs (a chunk of
 *     one or a few sequences) and when they are not a whole number of waves (256
 *     tiles of a 4 x 512-token chunk at 8K on 148 SMs: 341-347 us against 355 us).
 *     Without it (NULL, or too small) one CTA serves each query tile whole.  The contents are scratch; calls sharing one workspace must
 *     be ordered on one stream.  The result is the same either way up to fp32
 *     rounding.
 * pa_prefill_attention_workspace_bytes returns 0 when the balanced mode does not
 * apply to these sizes (the call then needs no workspace).
 * Host errors: B = 0 or max_q_len = 0 -> PA_OK; a NULL out, q, cu_q, pool, table,
 * ctx_lens or err_flag -> PA_ERR_NULL; max_q_len < 0, Hq not a positive multiple
 * of Hkv, G not a power of two up to 16, a NaN scale or sizes outside the
 * supported ranges -> PA_ERR_SHAPE; out, q, a pool or the workspace not 16-byte
 * aligned, or block_stride*2 not a multiple of 16 -> PA_ERR_ALIGN.
 * ==========================================================================*/
size_t pa_prefill_attention_workspace_bytes(int B, int Hq, int Hkv, int d, int bs, int max_q_len);

int pa_prefill_attention(uint16_t *out, const uint16_t *q, const int32_t *cu_q, int max_q_len,
                         const uint16_t *k_cache, const uint16_t *v_cache, int64_t block_stride,
                         const int32_t *block_tables, int max_blocks_per_seq,
                         const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs,
                         int64_t num_blocks, float scale, int32_t *err_flag, void *workspace,
                         size_t workspace_bytes, void *stream);

/* ============================================================================
 * Self-test of the device failure path (no counterpart in the pages).
 * Every pipeline wait in these kernels is bounded: after ~2 s of device time it
 * gives up, the kernel sets PA_DEV_TIMEOUT in err_flag and returns, and the CUDA
 * context stays usable.  This call launches one CTA whose wait (the same bounded
 * mbarrier wait the decode pipeline uses) is on a phase nothing completes, so it
 * takes that path: *err_flag (device int32, caller-zeroed) gets PA_DEV_TIMEOUT
 * after ~2 s.  No fault, trap or hang is involved.  Returns PA_OK or a PA_ERR_*
 * code (PA_ERR_NULL for a NULL flag).
 * ==========================================================================*/
int pa_selftest_wait_timeout(int32_t *err_flag, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* PAGEDKV_H */
