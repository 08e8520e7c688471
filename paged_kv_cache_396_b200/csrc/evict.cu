// evict.cu -- PagedEviction token importance and block selection
// (blog.hotdry.top "KV缓存内存布局优化", "PagedEviction 块级驱逐机制"):
//   S = ||V||_2 / ||K||_2 per (token, kv head), needing no attention weights;
//   in the decode phase the complete block with the lowest mean S is evicted.
#include <limits.h>
#include <math.h>

#include "blockmean.cuh"
#include "common.cuh"
#include "kernels.h"
#include "prefill.h"

namespace pkv {

__device__ __forceinline__ float norm_ratio(float kk, float vv) {
    if (kk == 0.f) return vv > 0.f ? INFINITY : 0.f;
    return sqrtf(vv) / sqrtf(kk);
}

// One CTA per (logical block j, sequence b).  A half-warp covers one (token,
// head) row of d elements with 16-byte loads (d = 128) or 8-byte loads
// (d = 64), so each row is one contiguous, coalesced read; the two halves of a
// warp take consecutive rows.
template <int D>
__global__ void __launch_bounds__(256) score_kernel(ScoreArgs a) {
    constexpr int PER = D / 16;  // bf16 elements per lane
    const int j = blockIdx.x, b = blockIdx.y;
    int len = a.ctx_lens[b];
    if (len < 0 || (int64_t)len > (int64_t)a.MB * a.bs) {
        if (j == 0 && threadIdx.x == 0) raise_flag(a.err, PA_DEV_BAD_LEN);
        return;
    }
    const int tbeg = j * a.bs;
    if (tbeg >= len) return;
    const int32_t phys = a.block_tables[(int64_t)b * a.MB + j];
    if (phys < 0 || (int64_t)phys >= a.N) {
        if (threadIdx.x == 0) raise_flag(a.err, PA_DEV_BAD_BLOCK);
        return;
    }
    const int ntok = min(a.bs, len - tbeg);
    const int rows = ntok * a.Hkv;
    const int half = threadIdx.x >> 4, sub = threadIdx.x & 15;
    const int halves = blockDim.x >> 4;
    const int64_t base = (int64_t)phys * a.block_stride;
    // every half-warp runs the same trip count so the shuffles see full warps
    const int trips = (rows + halves - 1) / halves;
    for (int it = 0; it < trips; ++it) {
        const int r = it * halves + half;
        const bool live = r < rows;
        float kk = 0.f, vv = 0.f;
        if (live) {
            const int64_t off = base + (int64_t)r * D + sub * PER;  // row r = slot*Hkv + h
            if constexpr (PER == 8) {
                const uint4 kw = __ldg(reinterpret_cast<const uint4 *>(a.k_cache + off));
                const uint4 vw = __ldg(reinterpret_cast<const uint4 *>(a.v_cache + off));
                const uint32_t ka[4] = {kw.x, kw.y, kw.z, kw.w};
                const uint32_t va[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float x = bf16_lo(ka[i]), y = bf16_hi(ka[i]);
                    kk = fmaf(x, x, kk); kk = fmaf(y, y, kk);
                    x = bf16_lo(va[i]); y = bf16_hi(va[i]);
                    vv = fmaf(x, x, vv); vv = fmaf(y, y, vv);
                }
            } else {
                const uint2 kw = __ldg(reinterpret_cast<const uint2 *>(a.k_cache + off));
                const uint2 vw = __ldg(reinterpret_cast<const uint2 *>(a.v_cache + off));
                const uint32_t ka[2] = {kw.x, kw.y};
                const uint32_t va[2] = {vw.x, vw.y};
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    float x = bf16_lo(ka[i]), y = bf16_hi(ka[i]);
                    kk = fmaf(x, x, kk); kk = fmaf(y, y, kk);
                    x = bf16_lo(va[i]); y = bf16_hi(va[i]);
                    vv = fmaf(x, x, vv); vv = fmaf(y, y, vv);
                }
            }
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
            kk += __shfl_xor_sync(0xffffffffu, kk, o);
            vv += __shfl_xor_sync(0xffffffffu, vv, o);
        }
        if (live && sub == 0) {
            const int t = tbeg + r / a.Hkv, h = r % a.Hkv;
            a.scores[((int64_t)b * a.MB * a.bs + t) * a.Hkv + h] = norm_ratio(kk, vv);
        }
    }
}

// One CTA per sequence, one warp per full block (blocks j = warp, warp + 32, ...):
// each block mean is an fp64 sum of its bs*Hkv fp32 scores divided by bs*Hkv;
// then a (mean, j) argmin with ties to the lowest j.
__global__ void __launch_bounds__(1024) select_evict_kernel(int32_t *evict, float *means,
                                                           const float *scores,
                                                           const int32_t *ctx_lens, int MB,
                                                           int Hkv, int bs) {
    const int b = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int len = ctx_lens[b];
    if (len < 0 || (int64_t)len > (int64_t)MB * bs) len = 0;
    const int nfull = len / bs;
    const int per = bs * Hkv;
    double best = INFINITY;
    int bj = INT_MAX;
    for (int j = warp; j < MB; j += nw) {
        if (j < nfull) {
            const double mean = warp_block_mean(scores + ((int64_t)b * MB + j) * per, per, lane);
            if (means && lane == 0) means[(int64_t)b * MB + j] = (float)mean;
            argmin_take(best, bj, mean, j);
        } else if (means && lane == 0) {
            means[(int64_t)b * MB + j] = __int_as_float(0x7fc00000);  // NaN: not a candidate
        }
    }
    const int win = cta_argmin(best, bj);
    if (threadIdx.x == 0) evict[b] = (nfull > 0 && win != INT_MAX) ? win : -1;
}

// Threshold policy: with the trigger on, every full block whose mean is below
// `thr` is marked, else the lowest-mean full block; with it off nothing is
// marked.  Means are written either way.
__global__ void __launch_bounds__(1024) select_threshold_kernel(
    uint8_t *mask, int32_t *count, float *means, const float *scores, const int32_t *ctx_lens,
    int MB, int Hkv, int bs, double thr, int triggered) {
    __shared__ int s_count;
    const int b = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    if (threadIdx.x == 0) s_count = 0;
    __syncthreads();
    int len = ctx_lens[b];
    if (len < 0 || (int64_t)len > (int64_t)MB * bs) len = 0;
    const int nfull = len / bs;
    const int per = bs * Hkv;
    double best = INFINITY;
    int bj = INT_MAX;
    for (int j = warp; j < MB; j += nw) {
        uint8_t below = 0;
        if (j < nfull) {
            const double mean = warp_block_mean(scores + ((int64_t)b * MB + j) * per, per, lane);
            if (means && lane == 0) means[(int64_t)b * MB + j] = (float)mean;
            argmin_take(best, bj, mean, j);
            below = triggered && mean < thr;
        } else if (means && lane == 0) {
            means[(int64_t)b * MB + j] = __int_as_float(0x7fc00000);
        }
        if (lane == 0) {
            mask[(int64_t)b * MB + j] = below;
            if (below) atomicAdd(&s_count, 1);
        }
    }
    const int win = cta_argmin(best, bj);  // its barriers also order the s_count adds
    if (threadIdx.x == 0) {
        int n = s_count;
        if (triggered && n == 0 && nfull > 0 && win != INT_MAX) {
            mask[(int64_t)b * MB + win] = 1;
            n = 1;
        }
        count[b] = n;
    }
}

cudaError_t launch_score(const ScoreArgs &a, cudaStream_t st) {
    dim3 grid(a.MB, a.B);
    if (a.d == 128) score_kernel<128><<<grid, 256, 0, st>>>(a);
    else score_kernel<64><<<grid, 256, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_select_evict(int32_t *evict, float *means, const float *scores,
                                const int32_t *ctx_lens, int B, int MB, int Hkv, int bs,
                                cudaStream_t st) {
    select_evict_kernel<<<B, 1024, 0, st>>>(evict, means, scores, ctx_lens, MB, Hkv, bs);
    return cudaGetLastError();
}

cudaError_t launch_select_threshold(uint8_t *mask, int32_t *count, float *means,
                                    const float *scores, const int32_t *ctx_lens, int B, int MB,
                                    int Hkv, int bs, double thr, int triggered, cudaStream_t st) {
    select_threshold_kernel<<<B, 1024, 0, st>>>(mask, count, means, scores, ctx_lens, MB, Hkv, bs,
                                               thr, triggered);
    return cudaGetLastError();
}

}  // namespace pkv
