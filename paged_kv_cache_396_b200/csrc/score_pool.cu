// score_pool.cu -- incremental PagedEviction scoring: the KV append also writes
// each new (token, kv head) importance S = ||V||_2 / ||K||_2 into a score pool
// that shares the KV pool's paging ([N][bs][Hkv] fp32), and the block selection
// reads the scores of full blocks through the block table.
//
// blog.hotdry.top "KV缓存内存布局优化", "PagedEviction 块级驱逐机制": the score
// needs only the token's own K and V, and in the decode phase a block is chosen
// only when the newest block fills -- so scoring each token once, when it is
// written, replaces a pass over the whole context with a pass over one score
// per (token, head).
#include <limits.h>
#include <math.h>

#include "blockmean.cuh"
#include "common.cuh"
#include "kernels.h"
#include "select_pooled.cuh"

namespace pkv {

__device__ __forceinline__ float ratio(float kk, float vv) {
    if (kk == 0.f) return vv > 0.f ? INFINITY : 0.f;
    return sqrtf(vv) / sqrtf(kk);
}

// One warp per (sequence, token, kv head) row: copy the D bf16 values of K and V
// into the pools (PER = D/32 per lane) and store the row's score.
template <int D>
__global__ void __launch_bounds__(256) append_scored_kernel(const uint16_t *__restrict__ k_new,
                                                            const uint16_t *__restrict__ v_new,
                                                            uint16_t *__restrict__ k_cache,
                                                            uint16_t *__restrict__ v_cache,
                                                            float *__restrict__ score_pool,
                                                            AppendArgs a) {
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)a.B * a.n_new * a.Hkv;
    const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < rows;
         row += warps) {
        const int h = (int)(row % a.Hkv);
        const int64_t bi = row / a.Hkv;
        const int i = (int)(bi % a.n_new);
        const int b = (int)(bi / a.n_new);
        const bool leader = (h == 0 && lane == 0);
        const int64_t pos = (int64_t)a.positions[b] + i;
        if (pos < 0 || pos >= (int64_t)a.MB * a.bs) {
            if (leader) {
                raise_flag(a.err, PA_DEV_BAD_LEN);
                if (a.slot_out) a.slot_out[bi] = -1;
            }
            continue;
        }
        const int32_t phys = a.block_tables[(int64_t)b * a.MB + pos / a.bs];
        if (phys < 0 || (int64_t)phys >= a.N) {
            if (leader) {
                raise_flag(a.err, PA_DEV_BAD_BLOCK);
                if (a.slot_out) a.slot_out[bi] = -1;
            }
            continue;
        }
        const int64_t off = pos % a.bs;
        const int64_t src = row * D + lane * PER;
        const int64_t dst = (int64_t)phys * a.block_stride + (off * a.Hkv + h) * D + lane * PER;
        float kk = 0.f, vv = 0.f;
        if constexpr (PER == 4) {
            const uint2 kw = __ldg(reinterpret_cast<const uint2 *>(k_new + src));
            const uint2 vw = __ldg(reinterpret_cast<const uint2 *>(v_new + src));
            *reinterpret_cast<uint2 *>(k_cache + dst) = kw;
            *reinterpret_cast<uint2 *>(v_cache + dst) = vw;
            const uint32_t ka[2] = {kw.x, kw.y}, va[2] = {vw.x, vw.y};
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float x = bf16_lo(ka[q]), y = bf16_hi(ka[q]);
                kk = fmaf(x, x, kk);
                kk = fmaf(y, y, kk);
                x = bf16_lo(va[q]);
                y = bf16_hi(va[q]);
                vv = fmaf(x, x, vv);
                vv = fmaf(y, y, vv);
            }
        } else {
            static_assert(PER == 2, "d must be 64 or 128");
            const uint32_t kw = __ldg(reinterpret_cast<const unsigned int *>(k_new + src));
            const uint32_t vw = __ldg(reinterpret_cast<const unsigned int *>(v_new + src));
            *reinterpret_cast<uint32_t *>(k_cache + dst) = kw;
            *reinterpret_cast<uint32_t *>(v_cache + dst) = vw;
            float x = bf16_lo(kw), y = bf16_hi(kw);
            kk = fmaf(x, x, fmaf(y, y, 0.f));
            x = bf16_lo(vw);
            y = bf16_hi(vw);
            vv = fmaf(x, x, fmaf(y, y, 0.f));
        }
        kk = warp_sum(kk);
        vv = warp_sum(vv);
        if (lane == 0) score_pool[((int64_t)phys * a.bs + off) * a.Hkv + h] = ratio(kk, vv);
        if (leader && a.slot_out) a.slot_out[bi] = (int64_t)phys * a.bs + off;
    }
}

// Block selection from the score pool: one CTA of kSelThreads threads per sequence
// (select_pooled.cuh).  256 threads keep the CTA small enough to run beside the
// decode kernel when the caller overlaps the two on two streams.
__global__ void __launch_bounds__(kSelThreads) select_pooled_kernel(
    int32_t *evict, float *means, const float *score_pool, const int32_t *block_tables,
    const int32_t *ctx_lens, int32_t *err, int MB, int Hkv, int bs, int64_t N) {
    select_pooled_cta(evict, means, score_pool, block_tables, ctx_lens, err, MB, Hkv, bs, N,
                      blockIdx.x);
}

cudaError_t launch_append_scored(const uint16_t *k_new, const uint16_t *v_new, uint16_t *k_cache,
                                 uint16_t *v_cache, float *score_pool, const AppendArgs &a,
                                 int num_sms, cudaStream_t st) {
    const int64_t rows = (int64_t)a.B * a.n_new * a.Hkv;
    const int threads = 256;
    int64_t blocks = (rows * 32 + threads - 1) / threads;
    blocks = blocks < (int64_t)num_sms * 16 ? blocks : (int64_t)num_sms * 16;
    if (a.d == 128)
        append_scored_kernel<128><<<(unsigned)blocks, threads, 0, st>>>(k_new, v_new, k_cache,
                                                                        v_cache, score_pool, a);
    else
        append_scored_kernel<64><<<(unsigned)blocks, threads, 0, st>>>(k_new, v_new, k_cache,
                                                                       v_cache, score_pool, a);
    return cudaGetLastError();
}

cudaError_t launch_select_pooled(int32_t *evict, float *means, const float *score_pool,
                                 const int32_t *block_tables, const int32_t *ctx_lens,
                                 int32_t *err, int B, int MB, int Hkv, int bs, int64_t N,
                                 cudaStream_t st) {
    select_pooled_kernel<<<B, kSelThreads, 0, st>>>(evict, means, score_pool, block_tables,
                                                    ctx_lens, err, MB, Hkv, bs, N);
    return cudaGetLastError();
}

}  // namespace pkv
