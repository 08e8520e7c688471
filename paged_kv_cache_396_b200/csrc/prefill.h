// prefill.h -- launchers of the PagedEviction prefill stage and of the
// block-table compactions (prefill.cu), and of the threshold eviction policy
// (evict.cu).  Argument checking happens in the C ABI entry points; these only
// launch.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pkv {

cudaError_t launch_prefill_scores(float *scores, const uint16_t *k, const uint16_t *v, int64_t T,
                                  int Hkv, int d, cudaStream_t stream);
cudaError_t launch_prefill_select(int32_t *keep_idx, int32_t *kept_len, const float *scores,
                                  const int32_t *cu, int B, int budget, int32_t *err,
                                  cudaStream_t stream);
cudaError_t launch_prefill_pack(uint16_t *k_cache, uint16_t *v_cache, int64_t block_stride,
                                const int32_t *bt, int MB, const uint16_t *k, const uint16_t *v,
                                const int32_t *cu, const int32_t *keep_idx,
                                const int32_t *kept_len, int B, int budget, int Hkv, int d,
                                int bs, int64_t N, int32_t *err, cudaStream_t stream);
cudaError_t launch_evict_compact(int32_t *bt, int MB, int32_t *ctx_lens, int32_t *freed,
                                 const int32_t *evict, int B, int bs, int32_t *err,
                                 cudaStream_t stream);

cudaError_t launch_evict_compact_mask(int32_t *bt, int MB, int32_t *ctx_lens, int32_t *freed,
                                      const uint8_t *mask, int B, int bs, int32_t *err,
                                      cudaStream_t stream);
cudaError_t launch_select_threshold(uint8_t *mask, int32_t *count, float *means,
                                    const float *scores, const int32_t *ctx_lens, int B, int MB,
                                    int Hkv, int bs, double thr, int triggered,
                                    cudaStream_t stream);

}  // namespace pkv
