/*
 * oracle.c -- plain, slow, fp64 CPU restatement of single-token paged decode
 * attention, the KV append, the PagedEviction norm-ratio score with its
 * block-mean argmin, and the symmetric INT8 KV quantiser.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this file:
 * only the tests, the smoke check and the benchmark's CPU-baseline leg load
 * it.  It shares no code, header, table or helper with the CUDA library.
 *
 * Sources (web pages, cited by title and section):
 *   [KVL]  blog.hotdry.top, "KV缓存内存布局优化：分页策略、量化压缩与动态驱逐的工程实践"
 *          (KV cache memory layout optimisation), sections "PagedAttention 分页策略"
 *          and "PagedEviction 块级驱逐机制".
 *   [VKV]  ybb.press, "LLM 推理 KV Cache 内存管理深度工程实践：从 PageAttention 到推测解码"
 *          (vLLM KV memory engineering notes), §1, §2.1 BlockTable, §2.2
 *          paged_attention_forward, §6.1 INT8 KV cache, §6.2 GQA.
 *   [NANO] blog.hotdry.top, nano-vLLM KV cache memory optimisation, section
 *          "物理内存布局：连续张量与分块策略" (the [2, L, blocks, bs, n_kv, d] tensor).
 *   [KVP]  t6page.pages.dev knowledge page "KV cache": eq. kv-per-token,
 *          eq. kv-llama3-8b, table tbl-kv-llama3-context, section
 *          "PagedAttention 的算子" (the operator).
 *
 * Layout conventions (shared with every caller, not with the CUDA code):
 *   pool  [N physical blocks][bs slots][Hkv heads][d]; block b starts at
 *         element b * block_stride (block_stride >= bs*Hkv*d).
 *   bt    [B][MB] int32 block table, logical block j of sequence b -> physical id.
 *   bf16 values are passed as their uint16 bit patterns.
 *
 * Readings where the pages are silent or inconsistent are stated at each
 * function.  Floating point: fp64 everywhere except the INT8 quantiser, which
 * the configuration fixes to one fp32 scale per (token, kv head) and which is
 * therefore restated in fp32 so that its integer codes are decided in the same
 * precision as any fp32 implementation.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared (see build.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Thread count of the parallel loops below (timing only; results do not depend
 * on it: every parallel loop writes disjoint outputs). */
void or_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* bf16 is the upper half of an IEEE binary32: widen by a 16-bit shift. */
static float bf16_to_f32(uint16_t x) {
    uint32_t u = ((uint32_t)x) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static double bf16_to_f64(uint16_t x) { return (double)bf16_to_f32(x); }

/* ------------------------------------------------------------------------ */
/* Sizes                                                                     */
/* ------------------------------------------------------------------------ */

/* KV bytes per token: one K and one V vector per layer and kv head.
 * [KVP] eq. kv-per-token: 2 * L * n_kv * d_head * bytes; [VKV] §1 states the
 * same product (2 x num_layers x num_kv_heads x head_dim x dtype_size). */
int64_t or_kv_bytes_per_token(int64_t L, int64_t n_kv, int64_t d, int64_t elt_bytes) {
    return 2 * L * n_kv * d * elt_bytes;
}

/* Blocks a sequence of len tokens occupies: ceil(len / bs).
 * [VKV] §2.1 BlockTable.allocate; [VKV] §2.2 loop bound; [KVP] KVCachePool. */
int64_t or_num_blocks(int64_t len, int64_t bs) {
    if (len <= 0) return 0;
    return (len + bs - 1) / bs;
}

/* Global slot of token position pos: the physical block holding logical block
 * pos/bs, times bs, plus the offset pos%bs inside it.
 * [VKV] §2.1 BlockTable.append_slot returns last_block*block_size+used_slots,
 * i.e. the same formula for the token that lands in the last block. */
int64_t or_slot(const int32_t *bt_row, int64_t pos, int64_t bs) {
    return (int64_t)bt_row[pos / bs] * bs + pos % bs;
}

/* ------------------------------------------------------------------------ */
/* KV append                                                                 */
/* ------------------------------------------------------------------------ */

/* Write n_new tokens per sequence into the pool: token i of sequence b goes to
 * position positions[b] + i, i.e. to slot or_slot(bt[b], pos, bs), head h.
 * k_new, v_new: [B][n_new][Hkv][d] bf16 bits.  slot_out (nullable): [B][n_new].
 * [VKV] §2.1 append_slot; [KVL] "PagedAttention 分页策略" (blocks are filled as
 * tokens are generated). */
void or_append_kv(const uint16_t *k_new, const uint16_t *v_new,
                  uint16_t *k_cache, uint16_t *v_cache, int64_t block_stride,
                  const int32_t *bt, int MB, const int32_t *positions,
                  int B, int n_new, int Hkv, int d, int bs, int64_t *slot_out) {
    for (int b = 0; b < B; ++b) {
        for (int i = 0; i < n_new; ++i) {
            int64_t pos = (int64_t)positions[b] + i;
            int64_t slot = or_slot(bt + (int64_t)b * MB, pos, bs);
            if (slot_out) slot_out[(int64_t)b * n_new + i] = slot;
            int64_t phys = slot / bs, off = slot % bs;
            for (int h = 0; h < Hkv; ++h) {
                int64_t dst = phys * block_stride + (off * Hkv + h) * (int64_t)d;
                int64_t src = (((int64_t)b * n_new + i) * Hkv + h) * (int64_t)d;
                memcpy(k_cache + dst, k_new + src, (size_t)d * sizeof(uint16_t));
                memcpy(v_cache + dst, v_new + src, (size_t)d * sizeof(uint16_t));
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Attention                                                                 */
/* ------------------------------------------------------------------------ */

/* Gather sequence b's first len tokens, in logical order, into contiguous fp64
 * K[len][Hkv][d] and V[len][Hkv][d].  Slots of the last block at or beyond len
 * are not read ([VKV] §2.2 valid_slots).  The source values are produced by
 * `load(pool, index, aux)`, so that bf16 and dequantised INT8 pools share it. */
typedef double (*load_fn)(const void *pool, const void *aux, int64_t idx, int64_t row, int Hd);

static double load_bf16(const void *pool, const void *aux, int64_t idx, int64_t row, int Hd) {
    (void)aux; (void)row; (void)Hd;
    return bf16_to_f64(((const uint16_t *)pool)[idx]);
}

/* INT8: value = scale[token row, head] * code, the dequantisation of [VKV] §6.1. */
static double load_int8(const void *pool, const void *aux, int64_t idx, int64_t row, int Hd) {
    (void)Hd;
    const float *scale = (const float *)aux;
    return (double)scale[row] * (double)((const int8_t *)pool)[idx];
}

static void gather_seq(double *Kc, double *Vc, const void *k_cache, const void *v_cache,
                       const void *k_aux, const void *v_aux, load_fn load,
                       int64_t block_stride, int64_t scale_block_stride,
                       const int32_t *bt_row, int len, int Hkv, int d, int bs) {
    for (int t = 0; t < len; ++t) {
        int64_t phys = bt_row[t / bs];
        int64_t off = t % bs;
        for (int h = 0; h < Hkv; ++h) {
            int64_t base = phys * block_stride + (off * Hkv + h) * (int64_t)d;
            int64_t srow = phys * scale_block_stride + off * Hkv + h; /* scale index */
            for (int e = 0; e < d; ++e) {
                Kc[((int64_t)t * Hkv + h) * d + e] = load(k_cache, k_aux, base + e, srow, Hkv * d);
                Vc[((int64_t)t * Hkv + h) * d + e] = load(v_cache, v_aux, base + e, srow, Hkv * d);
            }
        }
    }
}

/* Softmax attention of one query vector q[d] over len contiguous keys/values of
 * kv head h (row stride Hkv*d): s_t = scale * q.k_t; p = softmax(s) taken over
 * ALL len tokens at once ([KVP] "PagedAttention 的算子": the scaled dot product
 * and softmax are done after merging every block); o = sum_t p_t v_t.
 * Two passes, max-subtracted.  len == 0 gives o = 0 (nothing to attend to). */
static void attend_one(double *o, const double *q, const double *Kc, const double *Vc,
                       int len, int Hkv, int h, int d, double scale, double *s) {
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    if (len <= 0) return;
    double m = -INFINITY;
    for (int t = 0; t < len; ++t) {
        const double *k = Kc + ((int64_t)t * Hkv + h) * d;
        double acc = 0.0;
        for (int e = 0; e < d; ++e) acc += q[e] * k[e];
        s[t] = scale * acc;
        if (s[t] > m) m = s[t];
    }
    double z = 0.0;
    for (int t = 0; t < len; ++t) {
        s[t] = exp(s[t] - m);
        z += s[t];
    }
    for (int t = 0; t < len; ++t) {
        const double *v = Vc + ((int64_t)t * Hkv + h) * d;
        double p = s[t] / z;
        for (int e = 0; e < d; ++e) o[e] += p * v[e];
    }
}

/* Shared body of the bf16 and INT8 decode oracles.
 * For every sequence b: gather its len_b = ctx_lens[b] tokens, then for every
 * query head i use kv head h = i / G with G = Hq / Hkv (contiguous GQA groups,
 * [VKV] §6.2: every G query heads share one KV group), and attend.
 * Lengths outside [0, MB*bs] are treated as 0 (output zero), as is len 0. */
static void decode_common(double *out, const uint16_t *q, const void *k_cache,
                          const void *v_cache, const void *k_aux, const void *v_aux,
                          load_fn load, int64_t block_stride, int64_t scale_block_stride,
                          const int32_t *bt, int MB, const int32_t *ctx_lens, int B,
                          int Hq, int Hkv, int d, int bs, double scale) {
    int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        int len = ctx_lens[b];
        if (len < 0 || (int64_t)len > (int64_t)MB * bs) len = 0;
        double *Kc = (double *)malloc(sizeof(double) * ((size_t)len * Hkv * d + 1));
        double *Vc = (double *)malloc(sizeof(double) * ((size_t)len * Hkv * d + 1));
        double *s = (double *)malloc(sizeof(double) * ((size_t)len + 1));
        double *qv = (double *)malloc(sizeof(double) * (size_t)d);
        gather_seq(Kc, Vc, k_cache, v_cache, k_aux, v_aux, load, block_stride,
                   scale_block_stride, bt + (int64_t)b * MB, len, Hkv, d, bs);
        for (int i = 0; i < Hq; ++i) {
            for (int e = 0; e < d; ++e) qv[e] = bf16_to_f64(q[((int64_t)b * Hq + i) * d + e]);
            attend_one(out + ((int64_t)b * Hq + i) * d, qv, Kc, Vc, len, Hkv, i / G, d, scale, s);
        }
        free(Kc); free(Vc); free(s); free(qv);
    }
}

/* Paged decode attention, bf16 pool.  out [B][Hq][d] fp64; q [B][Hq][d] bf16.
 * [VKV] §2.2 paged_attention_forward (query, paged cache, block table, context
 * length, scale), batched over sequences; separate K and V pools ([NANO]
 * index 0 = key, 1 = value), softmax over the whole context ([KVP] operator). */
void or_paged_decode(double *out, const uint16_t *q, const uint16_t *k_cache,
                     const uint16_t *v_cache, int64_t block_stride, const int32_t *bt,
                     int MB, const int32_t *ctx_lens, int B, int Hq, int Hkv, int d,
                     int bs, double scale) {
    decode_common(out, q, k_cache, v_cache, NULL, NULL, load_bf16, block_stride, 0, bt, MB,
                  ctx_lens, B, Hq, Hkv, d, bs, scale);
}

/* Paged decode attention over an INT8 pool: every element is dequantised as
 * scale[token, head] * code ([VKV] §6.1) before the same fp64 attention.
 * Scale pools are [N][bs][Hkv] fp32 (block stride bs*Hkv). */
void or_paged_decode_int8(double *out, const uint16_t *q, const int8_t *kq, const int8_t *vq,
                          const float *k_scale, const float *v_scale, int64_t block_stride,
                          const int32_t *bt, int MB, const int32_t *ctx_lens, int B, int Hq,
                          int Hkv, int d, int bs, double scale) {
    decode_common(out, q, kq, vq, k_scale, v_scale, load_int8, block_stride,
                  (int64_t)bs * Hkv, bt, MB, ctx_lens, B, Hq, Hkv, d, bs, scale);
}

/* ------------------------------------------------------------------------ */
/* PagedEviction                                                             */
/* ------------------------------------------------------------------------ */

/* Token importance S = ||V||_2 / ||K||_2 over the d elements of one (token,
 * kv head) vector ([KVL] "PagedEviction 块级驱逐机制": the ratio of the value and
 * key L2 norms, no attention weights needed).  Reading: the pages give one
 * S_i per token with no head index; here it is per (token, kv head).
 * ||K|| = 0: S = +inf when ||V|| > 0, else 0. */
static double norm_ratio(double kk, double vv) {
    if (kk == 0.0) return vv > 0.0 ? INFINITY : 0.0;
    return sqrt(vv) / sqrt(kk);
}

static void score_common(double *scores, const void *k_cache, const void *v_cache,
                         const void *k_aux, const void *v_aux, load_fn load,
                         int64_t block_stride, int64_t scale_block_stride, const int32_t *bt,
                         int MB, const int32_t *ctx_lens, int B, int Hkv, int d, int bs) {
    int64_t T = (int64_t)MB * bs;
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        int len = ctx_lens[b];
        if (len < 0 || (int64_t)len > T) len = 0;
        for (int t = 0; t < len; ++t) {
            int64_t phys = bt[(int64_t)b * MB + t / bs];
            int64_t off = t % bs;
            for (int h = 0; h < Hkv; ++h) {
                int64_t base = phys * block_stride + (off * Hkv + h) * (int64_t)d;
                int64_t srow = phys * scale_block_stride + off * Hkv + h;
                double kk = 0.0, vv = 0.0;
                for (int e = 0; e < d; ++e) {
                    double k = load(k_cache, k_aux, base + e, srow, Hkv * d);
                    double v = load(v_cache, v_aux, base + e, srow, Hkv * d);
                    kk += k * k;
                    vv += v * v;
                }
                scores[((int64_t)b * T + t) * Hkv + h] = norm_ratio(kk, vv);
            }
        }
    }
}

/* scores [B][MB*bs][Hkv] fp64; entries with t >= len_b are left untouched. */
void or_score_tokens(double *scores, const uint16_t *k_cache, const uint16_t *v_cache,
                     int64_t block_stride, const int32_t *bt, int MB, const int32_t *ctx_lens,
                     int B, int Hkv, int d, int bs) {
    score_common(scores, k_cache, v_cache, NULL, NULL, load_bf16, block_stride, 0, bt, MB,
                 ctx_lens, B, Hkv, d, bs);
}

/* Same score over the dequantised INT8 values. */
void or_score_tokens_int8(double *scores, const int8_t *kq, const int8_t *vq,
                          const float *k_scale, const float *v_scale, int64_t block_stride,
                          const int32_t *bt, int MB, const int32_t *ctx_lens, int B, int Hkv,
                          int d, int bs) {
    score_common(scores, kq, vq, k_scale, v_scale, load_int8, block_stride, (int64_t)bs * Hkv,
                 bt, MB, ctx_lens, B, Hkv, d, bs);
}

/* Decode-phase block eviction ([KVL] "PagedEviction 块级驱逐机制": when the
 * newest block is full, average the importance of every existing block and
 * evict the complete block with the lowest mean; eviction is always whole
 * blocks).  Reading: candidates are the full logical blocks j < floor(len/bs);
 * mean_j = sum of S over the bs*Hkv (token, head) entries of block j, divided
 * by bs*Hkv; ties go to the lowest j; no full block gives -1.
 * scores [B][MB*bs][Hkv] fp64 (an fp32 score array widened to fp64 is exact);
 * evict [B]; means (nullable) [B][MB], entries of non-candidate blocks set to
 * NAN; gap (nullable) [B] = second-lowest minus lowest mean (+inf when fewer
 * than two candidates), the margin by which the decision is made. */
void or_select_evict_block(int32_t *evict, double *means, double *gap, const double *scores,
                           const int32_t *ctx_lens, int B, int MB, int Hkv, int bs) {
    int64_t T = (int64_t)MB * bs;
    for (int b = 0; b < B; ++b) {
        int len = ctx_lens[b];
        if (len < 0 || (int64_t)len > T) len = 0;
        int nfull = len / bs;
        int best = -1;
        double best_mean = INFINITY, second = INFINITY;
        for (int j = 0; j < MB; ++j) {
            if (j >= nfull) {
                if (means) means[(int64_t)b * MB + j] = NAN;
                continue;
            }
            double sum = 0.0;
            for (int t = j * bs; t < (j + 1) * bs; ++t)
                for (int h = 0; h < Hkv; ++h) sum += scores[((int64_t)b * T + t) * Hkv + h];
            double mean = sum / (double)(bs * Hkv);
            if (means) means[(int64_t)b * MB + j] = mean;
            if (best < 0 || mean < best_mean) {
                second = best_mean;
                best_mean = mean;
                best = j;
            } else if (mean < second) {
                second = mean;
            }
        }
        evict[b] = best;
        if (gap) gap[b] = (best < 0 || second == INFINITY) ? INFINITY : second - best_mean;
    }
}

/* ------------------------------------------------------------------------ */
/* INT8 quantiser                                                            */
/* ------------------------------------------------------------------------ */

/* Symmetric INT8 quantisation of rows of d bf16 values, fp32 arithmetic
 * ([VKV] §6.1 quantize_kv_cache: scale = amax(|x|, last dim) / 127,
 * code = round(x / scale) as int8).  Readings: the scale is fp32, one per
 * (token, kv head) row; round() is PyTorch's, i.e. half to even (rintf in the
 * default rounding mode); amax = 0 gives scale 0 and all codes 0.  Every step
 * is one correctly rounded IEEE binary32 operation.
 * x [rows][d] bf16 bits; codes [rows][d]; scales [rows]. */
void or_quantize_int8(const uint16_t *x, int64_t rows, int d, int8_t *codes, float *scales) {
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *xr = x + r * d;
        float amax = 0.0f;
        for (int e = 0; e < d; ++e) {
            float a = fabsf(bf16_to_f32(xr[e]));
            if (a > amax) amax = a;
        }
        volatile float s = amax / 127.0f; /* volatile: keep it a single fp32 division */
        scales[r] = s;
        for (int e = 0; e < d; ++e) {
            if (s == 0.0f) {
                codes[r * d + e] = 0;
            } else {
                volatile float y = bf16_to_f32(xr[e]) / s;
                codes[r * d + e] = (int8_t)(int)rintf(y);
            }
        }
    }
}

/* INT8 append: quantise token i of sequence b (each kv head row separately)
 * and store codes into slot or_slot(bt[b], positions[b]+i) and its scale into
 * the [N][bs][Hkv] scale pools. */
void or_append_kv_int8(const uint16_t *k_new, const uint16_t *v_new, int8_t *kq, int8_t *vq,
                       float *k_scale, float *v_scale, int64_t block_stride, const int32_t *bt,
                       int MB, const int32_t *positions, int B, int n_new, int Hkv, int d, int bs,
                       int64_t *slot_out) {
    for (int b = 0; b < B; ++b) {
        for (int i = 0; i < n_new; ++i) {
            int64_t pos = (int64_t)positions[b] + i;
            int64_t slot = or_slot(bt + (int64_t)b * MB, pos, bs);
            if (slot_out) slot_out[(int64_t)b * n_new + i] = slot;
            int64_t phys = slot / bs, off = slot % bs;
            for (int h = 0; h < Hkv; ++h) {
                int64_t src = (((int64_t)b * n_new + i) * Hkv + h) * (int64_t)d;
                int64_t dst = phys * block_stride + (off * Hkv + h) * (int64_t)d;
                int64_t sdst = (phys * bs + off) * Hkv + h;
                or_quantize_int8(k_new + src, 1, d, kq + dst, k_scale + sdst);
                or_quantize_int8(v_new + src, 1, d, vq + dst, v_scale + sdst);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* FP8 (e4m3) KV                                                             */
/* ------------------------------------------------------------------------ */

/* [VKV] §6.1: the FP8 branch of quantize_kv_cache casts the KV tensor to
 * float8_e4m3fn.  Format (OCP FP8 e4m3): 1 sign bit, 4 exponent bits with bias
 * 7, 3 mantissa bits; normal values 2^(E-7) * (1 + m/8), subnormals m * 2^-9;
 * largest finite value 448 (0x7e); 0x7f / 0xff are NaN; there is no infinity.
 * Reading: round to nearest, ties to even; finite values beyond 448 saturate to
 * +-448; NaN stays NaN. */
uint8_t or_f32_to_e4m3(float x) {
    if (x != x) return 0x7f;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a > 448.0) a = 448.0;
    if (a < ldexp(1.0, -6)) {                  /* subnormal range: steps of 2^-9 */
        const double m = rint(a * 512.0);      /* 8 lands exactly on 2^-6, code 0x08 */
        return (uint8_t)(sign | (uint8_t)m);
    }
    int e;
    frexp(a, &e);                              /* a = f * 2^e, f in [0.5, 1) */
    int E = e - 1;                             /* a in [2^E, 2^(E+1)) */
    double m = rint(a / ldexp(1.0, E - 3));    /* in [8, 16] */
    if (m == 16.0) {
        m = 8.0;
        E += 1;
    }
    return (uint8_t)(sign | (uint8_t)(((E + 7) << 3) | ((int)m - 8)));
}

double or_e4m3_to_f64(uint8_t c) {
    const int s = c >> 7, E = (c >> 3) & 15, m = c & 7;
    if ((c & 0x7f) == 0x7f) return NAN;
    const double v = E == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, E - 7);
    return s ? -v : v;
}

void or_quantize_e4m3(const uint16_t *x, int64_t n, uint8_t *codes) {
    for (int64_t i = 0; i < n; ++i) codes[i] = or_f32_to_e4m3(bf16_to_f32(x[i]));
}

/* FP8 append: the new rows are cast to e4m3 and stored at their slots. */
void or_append_kv_fp8(const uint16_t *k_new, const uint16_t *v_new, uint8_t *k_cache,
                      uint8_t *v_cache, int64_t block_stride, const int32_t *bt, int MB,
                      const int32_t *positions, int B, int n_new, int Hkv, int d, int bs,
                      int64_t *slot_out) {
    for (int b = 0; b < B; ++b) {
        for (int i = 0; i < n_new; ++i) {
            int64_t pos = (int64_t)positions[b] + i;
            int64_t slot = or_slot(bt + (int64_t)b * MB, pos, bs);
            if (slot_out) slot_out[(int64_t)b * n_new + i] = slot;
            int64_t phys = slot / bs, off = slot % bs;
            for (int h = 0; h < Hkv; ++h) {
                int64_t src = (((int64_t)b * n_new + i) * Hkv + h) * (int64_t)d;
                int64_t dst = phys * block_stride + (off * Hkv + h) * (int64_t)d;
                or_quantize_e4m3(k_new + src, d, k_cache + dst);
                or_quantize_e4m3(v_new + src, d, v_cache + dst);
            }
        }
    }
}

static double load_fp8(const void *pool, const void *aux, int64_t idx, int64_t row, int Hd) {
    (void)aux; (void)row; (void)Hd;
    return or_e4m3_to_f64(((const uint8_t *)pool)[idx]);
}

/* Paged decode attention over e4m3 pools (each element decoded exactly). */
void or_paged_decode_fp8(double *out, const uint16_t *q, const uint8_t *k_cache,
                         const uint8_t *v_cache, int64_t block_stride, const int32_t *bt, int MB,
                         const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs,
                         double scale) {
    decode_common(out, q, k_cache, v_cache, NULL, NULL, load_fp8, block_stride, 0, bt, MB,
                  ctx_lens, B, Hq, Hkv, d, bs, scale);
}

/* ------------------------------------------------------------------------ */
/* PagedEviction prefill stage and block-table compaction                    */
/* ------------------------------------------------------------------------ */

/* Prefill token importance ([KVL] "PagedEviction 块级驱逐机制", the two-stage
 * strategy: at prefill every token is scored and the lowest-scoring tokens are
 * evicted down to the cache budget).  Reading: one slot holds a token for all
 * kv heads, so a token is kept or evicted as a whole and its importance is the
 * mean over the Hkv heads of the per-head ratio ||V||/||K|| (zero rule as in
 * norm_ratio); this is the same per-entry average the decode-phase block mean
 * takes.  k, v [T][Hkv][d] bf16 bits (the prompt rows, token-major); scores [T]. */
void or_prefill_scores(double *scores, const uint16_t *k, const uint16_t *v, int64_t T, int Hkv,
                       int d) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double sum = 0.0;
        for (int h = 0; h < Hkv; ++h) {
            const int64_t base = (t * Hkv + h) * (int64_t)d;
            double kk = 0.0, vv = 0.0;
            for (int e = 0; e < d; ++e) {
                const double x = bf16_to_f64(k[base + e]), y = bf16_to_f64(v[base + e]);
                kk += x * x;
                vv += y * y;
            }
            sum += norm_ratio(kk, vv);
        }
        scores[t] = sum / (double)Hkv;
    }
}

/* Value order used by the keep decision: numeric, NaN counted as -inf, -0 equal
 * to +0; equal values are ordered by token index, the later token ranking higher. */
static double rank_value(double x) { return x != x ? -INFINITY : x; }

typedef struct {
    double s;
    int32_t i;
} scored_token;

/* qsort comparator: best first (higher value, then higher index). */
static int best_first(const void *pa, const void *pb) {
    const scored_token *a = (const scored_token *)pa, *b = (const scored_token *)pb;
    if (a->s != b->s) return a->s > b->s ? -1 : 1;
    return a->i > b->i ? -1 : (a->i < b->i ? 1 : 0);
}

static int by_index(const void *pa, const void *pb) {
    const int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* Prefill keep set ([KVL] two-stage strategy, prefill side).  Readings: the
 * `budget` tokens that rank highest stay, all others are evicted; on equal
 * importance the earlier token goes first (the decode-side argmin also takes the
 * lowest index on ties); a prompt of n <= budget tokens keeps every token; kept
 * tokens keep their prompt order.
 * scores: one value per prompt token, prompts concatenated; cu [B+1] offsets;
 * keep_idx [B][budget]: prompt-local index of the p-th kept token, -1 after the
 * last; kept_len [B] = min(n_b, budget). */
void or_prefill_select(int32_t *keep_idx, int32_t *kept_len, const double *scores,
                       const int32_t *cu, int B, int budget) {
    for (int b = 0; b < B; ++b) {
        const int n = cu[b + 1] - cu[b];
        const int kept = n < budget ? n : budget;
        scored_token *tok = (scored_token *)malloc(sizeof(scored_token) * (size_t)(n > 0 ? n : 1));
        for (int i = 0; i < n; ++i) {
            tok[i].s = rank_value(scores[cu[b] + i]);
            tok[i].i = i;
        }
        qsort(tok, (size_t)n, sizeof(scored_token), best_first);
        int32_t *row = keep_idx + (int64_t)b * budget;
        for (int p = 0; p < budget; ++p) row[p] = p < kept ? tok[p].i : -1;
        qsort(row, (size_t)kept, sizeof(int32_t), by_index);
        kept_len[b] = kept;
        free(tok);
    }
}

/* Packing the kept prompt tokens into the paged pool: the p-th kept token of
 * sequence b is written at position p through the block table ([VKV] §2.1,
 * slot = bt[b][p/bs]*bs + p%bs), so the compressed prompt fills its blocks
 * densely and only the last one may be partial.  k, v [T][Hkv][d] bf16 bits
 * (prompts concatenated, offsets cu); pools [N][bs][Hkv][d]. */
void or_prefill_pack(const uint16_t *k, const uint16_t *v, const int32_t *cu,
                     const int32_t *keep_idx, const int32_t *kept_len, int budget,
                     uint16_t *k_cache, uint16_t *v_cache, int64_t block_stride,
                     const int32_t *bt, int MB, int B, int Hkv, int d, int bs) {
    const int64_t row = (int64_t)Hkv * d;
    for (int b = 0; b < B; ++b) {
        for (int p = 0; p < kept_len[b]; ++p) {
            const int64_t src = ((int64_t)cu[b] + keep_idx[(int64_t)b * budget + p]) * row;
            const int64_t slot = or_slot(bt + (int64_t)b * MB, p, bs);
            const int64_t dst = (slot / bs) * block_stride + (slot % bs) * row;
            memcpy(k_cache + dst, k + src, (size_t)row * sizeof(uint16_t));
            memcpy(v_cache + dst, v + src, (size_t)row * sizeof(uint16_t));
        }
    }
}

/* Block-table compaction after a decode-phase eviction ([KVL]: eviction drops a
 * whole block, so no partially filled block is left behind).  Reading: logical
 * block j = evict[b] leaves sequence b's table, the entries after it move down
 * by one, the last used entry becomes -1, the context length drops by bs and the
 * freed physical id is returned in freed[b].  evict[b] < 0, or an index that is
 * not a full block, leaves the sequence unchanged (freed[b] = -1).  Physical blocks do not move, so the cached rows
 * and any per-slot data stay where they are. */
void or_evict_compact(int32_t *bt, int32_t *ctx_lens, int32_t *freed, const int32_t *evict,
                      int B, int MB, int bs) {
    for (int b = 0; b < B; ++b) {
        int32_t *row = bt + (int64_t)b * MB;
        const int j = evict[b];
        freed[b] = -1;
        if (j < 0 || j >= ctx_lens[b] / bs) continue;   /* only full blocks are candidates */
        const int nblk = (int)or_num_blocks(ctx_lens[b], bs);
        freed[b] = row[j];
        for (int x = j; x < nblk - 1; ++x) row[x] = row[x + 1];
        row[nblk - 1] = -1;
        ctx_lens[b] -= bs;
    }
}

/* Threshold eviction policy (blog.hotdry.top nano-vLLM KV cache page, section
 * "工程落地：参数配置与监控要点": eviction_ratio = 0.2 starts eviction once cache
 * usage passes 80 %, and blocks whose importance is below importance_threshold
 * are evicted first).  Readings: the trigger is used_blocks > (1 - eviction_ratio)
 * * total_blocks, evaluated in fp64 (below it nothing is evicted); once triggered,
 * every full block of a sequence whose mean importance (the decode-phase block
 * mean) is below importance_threshold is evicted, and a sequence with no such
 * block evicts its single lowest-mean full block (the decode-phase rule, ties to
 * the lowest index); a sequence with no full block evicts nothing.
 * scores [B][MB*bs][Hkv] fp64; mask [B][MB] (1 = evict); count [B]; means
 * (nullable) [B][MB] as in or_select_evict_block. */
void or_select_evict_threshold(uint8_t *mask, int32_t *count, double *means,
                               const double *scores, const int32_t *ctx_lens, int B, int MB,
                               int Hkv, int bs, int64_t used_blocks, int64_t total_blocks,
                               double eviction_ratio, double importance_threshold) {
    const int triggered = (double)used_blocks > (1.0 - eviction_ratio) * (double)total_blocks;
    double *m = (double *)malloc(sizeof(double) * (size_t)B * (size_t)MB);
    int32_t *argmin = (int32_t *)malloc(sizeof(int32_t) * (size_t)(B > 0 ? B : 1));
    or_select_evict_block(argmin, m, NULL, scores, ctx_lens, B, MB, Hkv, bs);
    for (int b = 0; b < B; ++b) {
        int n = 0;
        for (int j = 0; j < MB; ++j) {
            const double mj = m[(int64_t)b * MB + j];
            const int below = triggered && mj == mj && mj < importance_threshold;
            mask[(int64_t)b * MB + j] = (uint8_t)below;
            n += below;
        }
        if (triggered && n == 0 && argmin[b] >= 0) {
            mask[(int64_t)b * MB + argmin[b]] = 1;
            n = 1;
        }
        count[b] = n;
    }
    if (means) memcpy(means, m, sizeof(double) * (size_t)B * (size_t)MB);
    free(m);
    free(argmin);
}

/* Table compaction for several evicted blocks per sequence: the full blocks
 * marked in mask[b] leave the table, the remaining entries keep their order and
 * close up, the context length drops by bs per evicted block, and the freed
 * physical ids are listed in freed[b][0..] in logical order (-1 after the last).
 * A mark on a block that is not full is ignored. */
void or_evict_compact_mask(int32_t *bt, int32_t *ctx_lens, int32_t *freed, const uint8_t *mask,
                           int B, int MB, int bs) {
    for (int b = 0; b < B; ++b) {
        int32_t *row = bt + (int64_t)b * MB;
        int32_t *fr = freed + (int64_t)b * MB;
        const int len = ctx_lens[b];
        const int nfull = len / bs, nblk = (int)or_num_blocks(len, bs);
        int w = 0, nf = 0;
        for (int j = 0; j < nblk; ++j) {
            if (j < nfull && mask[(int64_t)b * MB + j]) fr[nf++] = row[j];
            else row[w++] = row[j];
        }
        for (int j = w; j < nblk; ++j) row[j] = -1;
        for (int j = nf; j < MB; ++j) fr[j] = -1;
        ctx_lens[b] = len - nf * bs;
    }
}

/* ------------------------------------------------------------------------ */
/* Multi-query paged attention (chunked prefill)                             */
/* ------------------------------------------------------------------------ */

/* Paged attention with several query tokens per sequence, as a chunked prefill
 * runs it (t6page "KV cache" page, "Chunked prefill：让 prefill 不阻塞 decode": a
 * long prompt is prefilled 512 tokens at a time, each chunk batched with the
 * running decodes; the operator is the paged attention of "PagedAttention 的算子"
 * and [VKV] §2.2 with more than one query row).  Readings: the chunk's own K/V
 * rows were appended before the call, so sequence b holds ctx_lens[b] tokens and
 * its q_len_b = cu_q[b+1] - cu_q[b] query tokens are the last q_len_b of them;
 * query token i of b sits at position p = ctx_lens[b] - q_len_b + i and attends
 * exactly the tokens t <= p (causal), softmax over all of them; q_len_b = 1 is
 * a decode step.  A sequence with q_len_b > ctx_lens[b] or a length outside
 * [0, MB*bs] is invalid and its output rows are zero.
 * q [Tq][Hq][d] bf16 (Tq = cu_q[B]); out [Tq][Hq][d] fp64. */
void or_paged_prefill(double *out, const uint16_t *q, const int32_t *cu_q,
                      const uint16_t *k_cache, const uint16_t *v_cache, int64_t block_stride,
                      const int32_t *bt, int MB, const int32_t *ctx_lens, int B, int Hq, int Hkv,
                      int d, int bs, double scale) {
    const int G = Hq / Hkv;
    for (int b = 0; b < B; ++b) {
        const int ql = cu_q[b + 1] - cu_q[b];
        int len = ctx_lens[b];
        const int bad = len < 0 || (int64_t)len > (int64_t)MB * bs || ql > len;
        if (bad) len = 0;
        double *Kc = (double *)malloc(sizeof(double) * ((size_t)len * Hkv * d + 1));
        double *Vc = (double *)malloc(sizeof(double) * ((size_t)len * Hkv * d + 1));
        gather_seq(Kc, Vc, k_cache, v_cache, NULL, NULL, load_bf16, block_stride, 0,
                   bt + (int64_t)b * MB, len, Hkv, d, bs);
        /* every (query token, head) row is independent: rows in parallel */
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t ri = 0; ri < (int64_t)ql * Hq; ++ri) {
            const int r = (int)(ri / Hq), i = (int)(ri % Hq);
            const int64_t row = (int64_t)cu_q[b] + r;
            const int upto = bad ? 0 : len - ql + r + 1;   /* tokens 0 .. p */
            double *s = (double *)malloc(sizeof(double) * ((size_t)len + 1));
            double *qv = (double *)malloc(sizeof(double) * (size_t)d);
            for (int e = 0; e < d; ++e) qv[e] = bf16_to_f64(q[(row * Hq + i) * d + e]);
            attend_one(out + (row * Hq + i) * d, qv, Kc, Vc, upto, Hkv, i / G, d, scale, s);
            free(s);
            free(qv);
        }
        free(Kc);
        free(Vc);
    }
}
