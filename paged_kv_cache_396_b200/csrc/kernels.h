// kernels.h -- argument blocks and launchers shared between the C-ABI layer
// (pagedkv_api.cu) and the kernel translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pkv {

// Element type of the KV pools.
enum KvType : int { kKvBf16 = 0, kKvInt8 = 1, kKvFp8 = 2 };

struct AppendArgs {
    const int32_t *block_tables;
    const int32_t *positions;
    int64_t *slot_out;
    int32_t *err;
    int64_t block_stride;  // elements between physical blocks of the pool
    int64_t N;             // physical blocks in the pool
    int B, n_new, Hkv, d, bs, MB;
};

// Header at the start of the staged decode's workspace, written by its plan
// kernel: unit counter, unit count, partition size chosen, the count of decode
// CTAs that finished taking units (the last one resets both counters, so a plan
// serves several decode calls), and the signature of the sizes it was made for.
struct TcHeader {
    unsigned counter;
    int n_units;
    int chunk;
    unsigned done;
    unsigned long long sig;
    int pad[58];
};
static_assert(sizeof(TcHeader) == 256, "TcHeader is the workspace's 256-byte header");

// Launch plan of one decode call, decided on the host from the sizes alone.
struct DecodePlan {
    int kernel;         // 0: general-shape kernel, 1: staged tensor-core kernel
    int S;              // partition slots per sequence
    int chunk;          // general: tokens per partition; staged: minimum tokens per partition
    int wph;            // staged: consumer warps per kv head (8 / Hkv) = partial slots per unit
    int tpw;            // staged: 16-token sub-tiles per consumer warp per stage
    int n_sub;          // staged: 16-token sub-tiles per stage (wph * tpw)
    int nstage, stage_bytes, v_off, ks_off, vs_off, smem_bytes, grid, units_per_cta;
    int balanced;       // staged: 1 = every CTA takes an equal token range (automatic split)
    size_t off_hdr, off_ns, off_units, off_cta, off_first, off_starts, off_ml, off_acc, ws_total;
    unsigned long long sig;  // staged: signature of the sizes the device plan is made for
};

// Decode problem.  K/V element type is given by the launcher (bf16 or int8).
struct DecodeArgs {
    uint16_t *out;                // [B][Hq][d] bf16
    const uint16_t *q;            // [B][Hq][d] bf16
    const void *k_cache;          // pool base (bf16 or int8)
    const void *v_cache;
    const float *k_scale;         // INT8 only: [N][bs][Hkv]
    const float *v_scale;
    const int32_t *block_tables;  // [B][MB]
    const int32_t *ctx_lens;      // [B]
    int32_t *err;
    float *ws_acc;                // [B][Hq][S][d] partial numerators (S > 1)
    float *ws_ml;                 // [B][Hq][S][2] partial (max, sum), log2 domain
    int64_t block_stride;
    int64_t N;
    float scale_log2;             // scale * log2(e)
    int B, Hq, Hkv, G, d, bs, MB;
    int num_splits;               // S: partitions per sequence (1 = write out directly)
    int chunk;                    // tokens per partition (multiple of 16 when S > 1)
    void *ws;                     // workspace base
    DecodePlan plan;
    int reuse_plan;               // staged: the workspace already holds the plan (no plan launch)
    // optional, in the same call: the pooled block selection (pe_select_evict_block_pooled)
    int32_t *sel_evict;           // [B], or nullptr: no selection
    float *sel_means;             // [B][MB] block means, or nullptr
    const float *sel_scores;      // score pool [N][bs][Hkv] fp32
};

struct ScoreArgs {
    float *scores;
    const uint16_t *k_cache;
    const uint16_t *v_cache;
    const int32_t *block_tables;
    const int32_t *ctx_lens;
    int32_t *err;
    int64_t block_stride;
    int64_t N;
    int B, Hkv, d, bs, MB;
};

cudaError_t launch_append_bf16(const uint16_t *k_new, const uint16_t *v_new, uint16_t *k_cache,
                               uint16_t *v_cache, const AppendArgs &a, int num_sms,
                               cudaStream_t stream);
cudaError_t launch_append_int8(const uint16_t *k_new, const uint16_t *v_new, int8_t *kq,
                               int8_t *vq, float *k_scale, float *v_scale, float *score_pool,
                               const AppendArgs &a, int num_sms, cudaStream_t stream);
cudaError_t launch_append_fp8(const uint16_t *k_new, const uint16_t *v_new, uint8_t *k8,
                              uint8_t *v8, const AppendArgs &a, int num_sms, cudaStream_t stream);
cudaError_t launch_append_scored(const uint16_t *k_new, const uint16_t *v_new, uint16_t *k_cache,
                                 uint16_t *v_cache, float *score_pool, const AppendArgs &a,
                                 int num_sms, cudaStream_t stream);
cudaError_t launch_select_pooled(int32_t *evict, float *means, const float *score_pool,
                                 const int32_t *block_tables, const int32_t *ctx_lens,
                                 int32_t *err, int B, int MB, int Hkv, int bs, int64_t N,
                                 cudaStream_t stream);

// Decode dispatch: the staged tensor-core kernel when the shape allows it,
// else the general-shape kernel; then the partition merge when S > 1.
cudaError_t launch_decode(const DecodeArgs &a, int kv, cudaStream_t stream);
// Staged kernel only: the plan kernel alone (writes the partition plan of
// a.ctx_lens into the workspace for later calls with reuse_plan set).
cudaError_t launch_decode_plan_only(const DecodeArgs &a, cudaStream_t stream);
cudaError_t launch_decode_simple(const DecodeArgs &a, int kv, cudaStream_t stream);
cudaError_t launch_decode_tc(const DecodeArgs &a, int kv, cudaStream_t stream);
DecodePlan make_decode_plan(int B, int Hq, int Hkv, int d, int bs, int MB, int num_splits,
                            int kv, int sms);
cudaError_t launch_merge(const DecodeArgs &a, cudaStream_t stream);

cudaError_t launch_score(const ScoreArgs &a, cudaStream_t stream);
cudaError_t launch_select_evict(int32_t *evict, float *means, const float *scores,
                                const int32_t *ctx_lens, int B, int MB, int Hkv, int bs,
                                cudaStream_t stream);

}  // namespace pkv
