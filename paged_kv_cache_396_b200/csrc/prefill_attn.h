// prefill_attn.h -- arguments and launcher of the multi-query (chunked prefill)
// paged attention kernel (prefill_attn.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pkv {

struct PrefillAttnArgs {
    uint16_t *out;                 // [Tq][Hq][d] bf16
    const uint16_t *q;             // [Tq][Hq][d] bf16
    const int32_t *cu_q;           // [B+1] query-token offsets
    const uint16_t *k_cache, *v_cache;
    int64_t block_stride;          // elements
    const int32_t *block_tables;   // [B][MB]
    const int32_t *ctx_lens;       // [B], the chunk included
    int32_t *err;
    int64_t N;
    int B, MB, Hq, Hkv, G, d, bs;
    float scale_log2;              // softmax scale * log2(e)
};

cudaError_t launch_prefill_attn(const PrefillAttnArgs &a, int max_q_len, cudaStream_t stream);

// tcgen05 / TMEM version (prefill_attn_tc.cu): d = 128, bs a multiple of 16.  With a
// workspace of prefill_attn_tc_workspace_bytes (0: no balanced mode for these sizes)
// the work is balanced over the SMs (one persistent CTA per SM, items cut at range
// boundaries, partial results merged); without it, one CTA per item.
bool prefill_attn_tc_supported(const PrefillAttnArgs &a);
size_t prefill_attn_tc_workspace_bytes(const PrefillAttnArgs &a, int max_q_len, int sms);
cudaError_t launch_prefill_attn_tc(const PrefillAttnArgs &a, int max_q_len, void *ws,
                                   size_t ws_bytes, int sms, cudaStream_t stream);

}  // namespace pkv
