// select_pooled.cuh -- the decode-phase PagedEviction block selection of one
// sequence from the paged score pool, as a CTA-wide device function, so that the
// stand-alone selection kernel and the decode's merge kernel (which can take the
// selection of every sequence in extra CTAs) run the same code.
//
// blog.hotdry.top "KV缓存内存布局优化", "PagedEviction 块级驱逐机制": the block with
// the lowest mean importance among the sequence's complete blocks is the one to
// evict; the scores of block j are the bs*Hkv contiguous scores of physical block
// block_tables[b][j] in a pool paged like the KV pool ([N][bs][Hkv] fp32).
#pragma once

#include <limits.h>
#include <math.h>

#include "blockmean.cuh"
#include "common.cuh"

namespace pkv {

constexpr int kSelThreads = 256;   // threads of a selection CTA

// Sequence b's evicted block (the lowest block mean, ties to the lowest j; -1 when
// the sequence has no full block) and, when means != nullptr, every block's mean
// (NaN for blocks that are not candidates).  Called by all kSelThreads threads of a
// CTA.  Each warp takes four consecutive full blocks at a time (j = 4 w .. 4 w + 3,
// then 4 * warps further) with their loads in flight together, reduced with the
// arithmetic of the selection over a [B][MB*bs][Hkv] score array, so both agree
// exactly on equal scores.
__device__ __forceinline__ void select_pooled_cta(int32_t *evict, float *means,
                                                  const float *score_pool,
                                                  const int32_t *block_tables,
                                                  const int32_t *ctx_lens, int32_t *err, int MB,
                                                  int Hkv, int bs, int64_t N, int b) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = kSelThreads >> 5;
    int len = ctx_lens[b];
    if (len < 0 || (int64_t)len > (int64_t)MB * bs) {
        if (threadIdx.x == 0) raise_flag(err, PA_DEV_BAD_LEN);
        len = 0;
    }
    const int nfull = len / bs;
    const int per = bs * Hkv;
    double best = INFINITY;
    int bj = INT_MAX;
    for (int j0 = 4 * warp; j0 < MB; j0 += 4 * nw) {
        const float *p[4] = {nullptr, nullptr, nullptr, nullptr};
        bool cand[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = j0 + i;
            cand[i] = j < nfull;
            if (cand[i]) {
                const int32_t phys = block_tables[(int64_t)b * MB + j];
                if (phys < 0 || (int64_t)phys >= N) {
                    if (lane == 0) raise_flag(err, PA_DEV_BAD_BLOCK);
                    cand[i] = false;
                } else {
                    p[i] = score_pool + (int64_t)phys * per;
                }
            }
        }
        double mean[4] = {0.0, 0.0, 0.0, 0.0};
        if (cand[0] || cand[1] || cand[2] || cand[3])   // warp-uniform
            warp_block_mean4(p, per, lane, mean);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = j0 + i;
            if (cand[i]) argmin_take(best, bj, mean[i], j);
            if (means && lane == 0 && j < MB)
                means[(int64_t)b * MB + j] = cand[i] ? (float)mean[i] : __int_as_float(0x7fc00000);
        }
    }
    const int win = cta_argmin(best, bj);
    if (threadIdx.x == 0) evict[b] = (nfull > 0 && win != INT_MAX) ? win : -1;
}

}  // namespace pkv
