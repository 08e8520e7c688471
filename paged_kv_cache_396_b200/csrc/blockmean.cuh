// blockmean.cuh -- the decode-phase block mean of PagedEviction (blog.hotdry.top
// "KV缓存内存布局优化", "PagedEviction 块级驱逐机制": the mean importance of
// every complete block), computed by one warp per block.
#pragma once

#include <cuda_runtime.h>
#include <limits.h>
#include <stdint.h>

namespace pkv {

// Mean of the `per` fp32 scores at p (bs*Hkv entries of one block): coalesced
// loads issued four at a time (independent, so their latencies overlap), fp64
// partial sums per lane, butterfly reduction.  Every lane returns the same value.
__device__ __forceinline__ double warp_block_mean(const float *__restrict__ p, int per,
                                                  int lane) {
    double s = 0.0;
    int k = lane;
    for (; k + 96 < per; k += 128) {
        const float a0 = __ldg(p + k), a1 = __ldg(p + k + 32);
        const float a2 = __ldg(p + k + 64), a3 = __ldg(p + k + 96);
        s += ((double)a0 + (double)a1) + ((double)a2 + (double)a3);
    }
    for (; k < per; k += 32) s += (double)__ldg(p + k);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s / (double)per;
}

// The means of up to four blocks at once (p[i] == nullptr: block i skipped, its
// out[i] untouched; at least one p[i] is set), each with exactly the arithmetic of
// warp_block_mean (the same values, bit for bit); the four blocks' loads are in
// flight together.
__device__ __forceinline__ void warp_block_mean4(const float *const (&p)[4], int per, int lane,
                                                 double (&out)[4]) {
    // skipped blocks read a set block's scores (their sums are discarded)
    const float *any = p[0] ? p[0] : p[1] ? p[1] : p[2] ? p[2] : p[3];
    double s[4] = {0.0, 0.0, 0.0, 0.0};
    int k = lane;
    for (; k + 96 < per; k += 128) {
        float a[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float *q = p[i] ? p[i] : any;
            a[i][0] = __ldg(q + k);
            a[i][1] = __ldg(q + k + 32);
            a[i][2] = __ldg(q + k + 64);
            a[i][3] = __ldg(q + k + 96);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
            s[i] += ((double)a[i][0] + (double)a[i][1]) + ((double)a[i][2] + (double)a[i][3]);
    }
    for (; k < per; k += 32) {
#pragma unroll
        for (int i = 0; i < 4; ++i) s[i] += (double)__ldg((p[i] ? p[i] : any) + k);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s[i] += __shfl_xor_sync(0xffffffffu, s[i], o);
        if (p[i]) out[i] = s[i] / (double)per;
    }
}

// (mean, j) argmin with ties to the lowest j; j = INT_MAX marks "none".
__device__ __forceinline__ void argmin_take(double &best, int &bj, double m, int j) {
    if (j != INT_MAX && (bj == INT_MAX || m < best || (m == best && j < bj))) {
        best = m;
        bj = j;
    }
}

// CTA-wide argmin of per-warp candidates (every lane of a warp holds its
// warp's candidate).  Returns the winner in every thread.
__device__ __forceinline__ int cta_argmin(double best, int bj) {
    __shared__ double sb[32];
    __shared__ int sj[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
        sb[warp] = best;
        sj[warp] = bj;
    }
    __syncthreads();
    double b = INFINITY;
    int j = INT_MAX;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) argmin_take(b, j, sb[w], sj[w]);
    __syncthreads();
    return j;
}

}  // namespace pkv
