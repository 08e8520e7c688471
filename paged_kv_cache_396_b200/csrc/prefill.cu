// prefill.cu -- the PagedEviction prefill stage and the block-table compaction
// that follows a decode-phase eviction.
//
// Source: blog.hotdry.top "KV缓存内存布局优化", section "PagedEviction 块级驱逐机制"
// (two-stage strategy: at prefill every token is scored with ||V||/||K|| and the
// lowest-scoring tokens are evicted down to the cache budget; at decode whole
// blocks are evicted, so no partially filled block is left behind).
//
//   prefill_score_kernel   one warp per prompt token: sums of squares of the
//                          token's K and V rows per kv head (16-byte loads,
//                          segmented shuffles), token score = head mean of the
//                          per-head norm ratio.  HBM-bound: reads every prompt
//                          row once.
//   prefill_select_kernel  one CTA per prompt: radix select (4 passes of 8 bits)
//                          of the budget-th highest score key, then an ordered
//                          compaction pass that writes the kept token indices in
//                          prompt order.  Reads the scores only (L2-resident).
//   prefill_pack_kernel    one warp per kept token: copies its K and V rows to
//                          position p of its sequence through the block table.
//   evict_compact_kernel   one warp per sequence: removes the evicted logical
//                          block from the table (entries after it move down by
//                          one), lowers the context length by bs, returns the
//                          freed physical id.
#include "common.cuh"
#include "kernels.h"
#include "prefill.h"

namespace pkv {

namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ void sumsq8(const uint4 w, float &acc) {
    const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float a = bf16_lo(x[i]), b = bf16_hi(x[i]);
        acc = fmaf(a, a, acc);
        acc = fmaf(b, b, acc);
    }
}

// Per-head ratio with the zero rule: ||K|| = 0 gives +inf when ||V|| > 0, else 0.
__device__ __forceinline__ float ratio(float kk, float vv) {
    if (kk == 0.f) return vv > 0.f ? INFINITY : 0.f;
    return sqrtf(vv) / sqrtf(kk);
}

// CPH = 16-byte chunks per head row (d / 8): a head's chunks are CPH adjacent
// lanes of one load round, so its sums come from a CPH-lane xor reduction.
template <int CPH>
__global__ void __launch_bounds__(256) prefill_score_kernel(float *__restrict__ scores,
                                                            const uint4 *__restrict__ k,
                                                            const uint4 *__restrict__ v,
                                                            int64_t T, int Hkv) {
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const int C = Hkv * CPH;  // chunks per token
    const uint4 *kr = k + t * C, *vr = v + t * C;
    float acc = 0.f;
    for (int c0 = 0; c0 < C; c0 += 128) {
        // up to four load rounds in flight before any arithmetic
        uint4 kw[4], vw[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int c = c0 + 32 * r + lane;
            kw[r] = c < C ? kr[c] : make_uint4(0, 0, 0, 0);
            vw[r] = c < C ? vr[c] : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            if (c0 + 32 * r >= C) break;  // warp-uniform
            float kk = 0.f, vv = 0.f;
            sumsq8(kw[r], kk);
            sumsq8(vw[r], vv);
#pragma unroll
            for (int o = CPH / 2; o > 0; o >>= 1) {
                kk += __shfl_xor_sync(kFull, kk, o);
                vv += __shfl_xor_sync(kFull, vv, o);
            }
            const int c = c0 + 32 * r + lane;
            if ((lane & (CPH - 1)) == 0 && c < C) acc += ratio(kk, vv);
        }
    }
    acc = warp_sum(acc);
    if (lane == 0) scores[t] = acc / (float)Hkv;
}

// Order-preserving map of a score to an unsigned key: numeric order, NaN
// counted as -inf, -0 equal to +0.
__device__ __forceinline__ uint32_t rank_key(float x) {
    if (x != x) x = -INFINITY;
    if (x == 0.f) x = 0.f;
    const uint32_t u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSelThreads = 1024;

// Exclusive prefix count of `flag` over the CTA (in thread order) and the
// CTA total.  Uses warp ballots and one shared array of warp counts.
__device__ __forceinline__ int cta_exclusive_count(bool flag, int *warp_cnt, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned m = __ballot_sync(kFull, flag);
    const int before_in_warp = __popc(m & ((1u << lane) - 1u));
    if (lane == 0) warp_cnt[warp] = __popc(m);
    __syncthreads();
    int before = 0, tot = 0;
    for (int w = 0; w < kSelThreads / 32; ++w) {
        const int c = warp_cnt[w];
        before += w < warp ? c : 0;
        tot += c;
    }
    __syncthreads();  // warp_cnt is reused by the next call
    total = tot;
    return before + before_in_warp;
}

__global__ void __launch_bounds__(kSelThreads) prefill_select_kernel(
    int32_t *__restrict__ keep_idx, int32_t *__restrict__ kept_len,
    const float *__restrict__ scores, const int32_t *__restrict__ cu, int budget,
    int32_t *err) {
    __shared__ uint32_t hist[256];
    __shared__ uint32_t s_digit, s_above, s_eq;
    __shared__ int warp_cnt[kSelThreads / 32];
    const int b = blockIdx.x, tid = threadIdx.x;
    const int64_t s0 = cu[b];
    int n = cu[b + 1] - cu[b];
    if (n < 0) {
        if (tid == 0) raise_flag(err, PA_DEV_BAD_LEN);
        n = 0;
    }
    int32_t *row = keep_idx + (int64_t)b * budget;
    if (n <= budget) {  // every token stays
        for (int p = tid; p < budget; p += kSelThreads) row[p] = p < n ? p : -1;
        if (tid == 0) kept_len[b] = n;
        return;
    }
    if (scores == nullptr) {  // no score array (no prompt tokens were given): keep nothing
        for (int p = tid; p < budget; p += kSelThreads) row[p] = -1;
        if (tid == 0) {
            kept_len[b] = 0;
            raise_flag(err, PA_DEV_BAD_LEN);
        }
        return;
    }
    const float *sc = scores + s0;
    // ---- radix select of the budget-th highest key, most significant digit first
    uint32_t prefix = 0, mask = 0;
    uint32_t rem = (uint32_t)budget;  // keys still to take at or below the current prefix
    uint32_t eq = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += kSelThreads) {
            const uint32_t key = rank_key(sc[i]);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            // warp scan from the top digit down: lane j owns digits 255-8j .. 248-8j
            uint32_t c[8], own = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                c[q] = hist[255 - 8 * tid - q];
                own += c[q];
            }
            uint32_t incl = own;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(kFull, incl, o);
                if (tid >= o) incl += y;
            }
            uint32_t run = incl - own;  // keys in digits above this lane's range
            if (run < rem && incl >= rem) {  // exactly one lane
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    if (run + c[q] >= rem) {
                        s_digit = 255u - 8u * tid - q;
                        s_above = run;
                        s_eq = c[q];
                        break;
                    }
                    run += c[q];
                }
            }
        }
        __syncthreads();
        const uint32_t dg = s_digit;
        rem -= s_above;
        eq = s_eq;
        prefix |= dg << shift;
        mask |= 255u << shift;
        __syncthreads();
    }
    // prefix is the threshold key; `rem` of the `eq` tokens equal to it stay,
    // the latest ones (ties evict the earlier token)
    const uint32_t tau = prefix;
    const int drop_ties = (int)(eq - rem);
    int base_tie = 0, base_keep = 0;
    for (int c0 = 0; c0 < n; c0 += kSelThreads) {
        const int i = c0 + tid;
        const uint32_t key = i < n ? rank_key(sc[i]) : 0u;
        const bool gt = i < n && key > tau, tie = i < n && key == tau;
        int tot_tie = 0, tot_keep = 0;
        const int tie_rank = base_tie + cta_exclusive_count(tie, warp_cnt, tot_tie);
        const bool keep = gt || (tie && tie_rank >= drop_ties);
        const int pos = base_keep + cta_exclusive_count(keep, warp_cnt, tot_keep);
        if (keep && pos < budget) row[pos] = i;
        base_tie += tot_tie;
        base_keep += tot_keep;
    }
    if (tid == 0) kept_len[b] = budget;
}

__global__ void __launch_bounds__(256) prefill_pack_kernel(
    uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache, int64_t block_stride16,
    const int32_t *__restrict__ bt, int MB, const uint4 *__restrict__ k,
    const uint4 *__restrict__ v, const int32_t *__restrict__ cu,
    const int32_t *__restrict__ keep_idx, const int32_t *__restrict__ kept_len, int B, int budget,
    int C, int bs, int64_t N, int32_t *err) {
    const int lane = threadIdx.x & 31;
    const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (w >= (int64_t)B * budget) return;
    const int b = (int)(w / budget), p = (int)(w % budget);
    if (p >= kept_len[b]) return;
    const int n = cu[b + 1] - cu[b];
    const int idx = keep_idx[w];
    const int j = p / bs;
    if (idx < 0 || idx >= n || j >= MB) {
        if (lane == 0) raise_flag(err, PA_DEV_BAD_LEN);
        return;
    }
    const int64_t blk = bt[(int64_t)b * MB + j];
    if (blk < 0 || blk >= N) {
        if (lane == 0) raise_flag(err, PA_DEV_BAD_BLOCK);
        return;
    }
    const int64_t src = ((int64_t)cu[b] + idx) * C;
    const int64_t dst = blk * block_stride16 + (int64_t)(p % bs) * C;
    for (int c = lane; c < C; c += 32) {
        k_cache[dst + c] = k[src + c];
        v_cache[dst + c] = v[src + c];
    }
}

__global__ void __launch_bounds__(128) evict_compact_kernel(int32_t *__restrict__ bt, int MB,
                                                            int32_t *__restrict__ ctx_lens,
                                                            int32_t *__restrict__ freed,
                                                            const int32_t *__restrict__ evict,
                                                            int B, int bs, int32_t *err) {
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (b >= B) return;
    const int j = evict[b];
    if (j < 0) {
        if (lane == 0 && freed) freed[b] = -1;
        return;
    }
    const int len = ctx_lens[b];
    if (len < 0 || (int64_t)len > (int64_t)MB * bs || j >= len / bs) {
        if (lane == 0) {
            raise_flag(err, len < 0 || (int64_t)len > (int64_t)MB * bs ? PA_DEV_BAD_LEN
                                                                         : PA_DEV_BAD_EVICT);
            if (freed) freed[b] = -1;
        }
        return;
    }
    const int nblk = (len + bs - 1) / bs;
    int32_t *row = bt + (int64_t)b * MB;
    const int32_t gone = row[j];
    __syncwarp();
    // shift entries j+1 .. nblk-1 down by one, 32 at a time in ascending order:
    // every entry is read (this round or the previous one) before it is overwritten
    for (int x0 = j; x0 < nblk - 1; x0 += 32) {
        const int x = x0 + lane;
        const int32_t val = x + 1 < nblk ? row[x + 1] : 0;
        __syncwarp();
        if (x < nblk - 1) row[x] = val;
        __syncwarp();
    }
    if (lane == 0) {
        row[nblk - 1] = -1;
        ctx_lens[b] = len - bs;
        if (freed) freed[b] = gone;
    }
}

// Several evicted blocks per sequence: the marked full blocks leave the table,
// the others close up in order.  One warp per sequence walks the table 32
// entries at a time; a ballot gives each survivor its new index and each
// evicted entry its place in the freed list.  Writes land at or below the
// entry being read and every round reads before it writes, so the compaction
// is in place.
__global__ void __launch_bounds__(128) evict_compact_mask_kernel(int32_t *__restrict__ bt,
                                                                 int MB,
                                                                 int32_t *__restrict__ ctx_lens,
                                                                 int32_t *__restrict__ freed,
                                                                 const uint8_t *__restrict__ mask,
                                                                 int B, int bs, int32_t *err) {
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (b >= B) return;
    const int len = ctx_lens[b];
    int32_t *row = bt + (int64_t)b * MB;
    int32_t *fr = freed ? freed + (int64_t)b * MB : nullptr;
    const uint8_t *mk = mask + (int64_t)b * MB;
    if (len < 0 || (int64_t)len > (int64_t)MB * bs) {
        if (lane == 0) raise_flag(err, PA_DEV_BAD_LEN);
        if (fr)
            for (int x = lane; x < MB; x += 32) fr[x] = -1;
        return;
    }
    const int nfull = len / bs, nblk = (len + bs - 1) / bs;
    const unsigned below = (1u << lane) - 1u;
    int w = 0, nf = 0;
    for (int x0 = 0; x0 < nblk; x0 += 32) {
        const int x = x0 + lane;
        const bool in = x < nblk;
        const int32_t val = in ? row[x] : 0;
        const bool marked = in && mk[x] != 0;
        const bool gone = marked && x < nfull;
        if (marked && !gone) raise_flag(err, PA_DEV_BAD_EVICT);  // a partial block: ignored
        const unsigned keep_m = __ballot_sync(kFull, in && !gone);
        const unsigned gone_m = __ballot_sync(kFull, gone);
        __syncwarp();
        if (in && !gone) row[w + __popc(keep_m & below)] = val;
        if (gone && fr) fr[nf + __popc(gone_m & below)] = val;
        w += __popc(keep_m);
        nf += __popc(gone_m);
        __syncwarp();
    }
    for (int x = w + lane; x < nblk; x += 32) row[x] = -1;
    if (fr)
        for (int x = nf + lane; x < MB; x += 32) fr[x] = -1;
    if (lane == 0) ctx_lens[b] = len - nf * bs;
}

}  // namespace

cudaError_t launch_evict_compact_mask(int32_t *bt, int MB, int32_t *ctx_lens, int32_t *freed,
                                      const uint8_t *mask, int B, int bs, int32_t *err,
                                      cudaStream_t st) {
    evict_compact_mask_kernel<<<(B + 3) / 4, 128, 0, st>>>(bt, MB, ctx_lens, freed, mask, B, bs,
                                                           err);
    return cudaGetLastError();
}

cudaError_t launch_prefill_scores(float *scores, const uint16_t *k, const uint16_t *v, int64_t T,
                                  int Hkv, int d, cudaStream_t st) {
    const int64_t blocks = (T + 7) / 8;
    const auto *k4 = reinterpret_cast<const uint4 *>(k);
    const auto *v4 = reinterpret_cast<const uint4 *>(v);
    switch (d) {
        case 64:
            prefill_score_kernel<8><<<(unsigned)blocks, 256, 0, st>>>(scores, k4, v4, T, Hkv);
            break;
        case 128:
            prefill_score_kernel<16><<<(unsigned)blocks, 256, 0, st>>>(scores, k4, v4, T, Hkv);
            break;
        case 256:
            prefill_score_kernel<32><<<(unsigned)blocks, 256, 0, st>>>(scores, k4, v4, T, Hkv);
            break;
        default:
            return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_prefill_select(int32_t *keep_idx, int32_t *kept_len, const float *scores,
                                  const int32_t *cu, int B, int budget, int32_t *err,
                                  cudaStream_t st) {
    prefill_select_kernel<<<B, kSelThreads, 0, st>>>(keep_idx, kept_len, scores, cu, budget, err);
    return cudaGetLastError();
}

cudaError_t launch_prefill_pack(uint16_t *k_cache, uint16_t *v_cache, int64_t block_stride,
                                const int32_t *bt, int MB, const uint16_t *k, const uint16_t *v,
                                const int32_t *cu, const int32_t *keep_idx,
                                const int32_t *kept_len, int B, int budget, int Hkv, int d,
                                int bs, int64_t N, int32_t *err, cudaStream_t st) {
    const int C = Hkv * d / 8;
    const int64_t warps = (int64_t)B * budget;
    const int64_t blocks = (warps + 7) / 8;
    prefill_pack_kernel<<<(unsigned)blocks, 256, 0, st>>>(
        reinterpret_cast<uint4 *>(k_cache), reinterpret_cast<uint4 *>(v_cache), block_stride / 8,
        bt, MB, reinterpret_cast<const uint4 *>(k), reinterpret_cast<const uint4 *>(v), cu,
        keep_idx, kept_len, B, budget, C, bs, N, err);
    return cudaGetLastError();
}

cudaError_t launch_evict_compact(int32_t *bt, int MB, int32_t *ctx_lens, int32_t *freed,
                                 const int32_t *evict, int B, int bs, int32_t *err,
                                 cudaStream_t st) {
    evict_compact_kernel<<<(B + 3) / 4, 128, 0, st>>>(bt, MB, ctx_lens, freed, evict, B, bs, err);
    return cudaGetLastError();
}

}  // namespace pkv
