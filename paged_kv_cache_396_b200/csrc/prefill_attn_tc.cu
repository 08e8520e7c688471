// prefill_attn_tc.cu -- multi-query (chunked prefill) paged attention on the
// fifth-generation tensor cores: tcgen05.mma with TMEM accumulators.
//
// Same operation as prefill_attn.cu (t6page.pages.dev "KV cache", "Chunked
// prefill：让 prefill 不阻塞 decode"; "PagedAttention 的算子"): the q_len query
// tokens of a sequence are its last q_len cached tokens and attend causally.
// Used for d = 128 and block sizes that are multiples of 16.
//
// One CTA = one (sequence, kv head, 256 query rows) as two tiles of 128 rows
// (the MMA M); rows are (query token, head of the GQA group) pairs, so each K/V
// tile serves all G heads of both Q tiles.  Warp roles (320 threads):
//   warps 0-3, 4-7  softmax, one warpgroup per Q tile: thread r owns row r of its
//              tile = TMEM lane r.  Loads its Q row into shared memory once; per
//              128-token K/V tile reads its S row from TMEM, masks (causal),
//              keeps the running max (lazy: O is rescaled only when the max grows
//              by more than 2^8), writes P = hi + lo (two bf16 parts) back over the
//              S columns, and at the end normalises O.  The two warpgroups work
//              half a step apart, so one computes softmax while the tensor core
//              runs the other tile's products.
//   warp 8     MMA issue (one lane), in the order PV_A(j), S_A(j+1), PV_B(j),
//              S_B(j+1): S = Q K^T (SS, both K-major) into the tile's S/P
//              columns, O += P_hi V + P_lo V (A from TMEM, V MN-major) into its O
//              columns; completion through tcgen05.commit.  Its lanes also zero
//              the V rows past the context end in a tile that holds them (stale or
//              NaN slots must not meet a zero weight).
//   warp 9     TMA producer: lane p < 8 owns 16-token page p of every tile, looks
//              up its physical block one tile ahead and issues four boxes (K and V,
//              two 64-element slices each); two stages.
// TMEM: S/P of tile A at columns [0,128), of tile B at [128,256); O of tile A at
// [256,384), of tile B at [384,512).
// Every mbarrier wait is bounded (2 s of globaltimer); a timeout sets
// PA_DEV_TIMEOUT and the CTA winds down, freeing its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "prefill_attn.h"
#include "ptx.cuh"

namespace pkv {

namespace {

constexpr int kD = 128;
constexpr int kM = 128;          // query rows per MMA tile (TMEM lanes)
constexpr int kRows = 2 * kM;    // query rows per CTA: two tiles
constexpr int kN = 128;          // tokens per K/V tile
constexpr int kThreads = 320;    // 8 softmax warps, 1 MMA warp, 1 TMA warp
constexpr int kSlice = kN * 128;         // one 64-element slice of a 128-row tile (bytes)
constexpr int kTileB = 2 * kSlice;       // a Q, K or V tile (d = 128)
constexpr int kStages = 2;       // K/V stages in flight
constexpr int kSmem = 2 * kTileB /*Q x 2*/ + kStages * 2 * kTileB /*K,V per stage*/ + 1024;
constexpr uint32_t kColO = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 2000000000ull;

// instruction descriptor: D f32, A/B bf16, M = 128, N = 128; B MN-major when mn
__host__ __device__ constexpr uint32_t idesc(bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn ? 1u : 0u) << 16) | ((kN / 8u) << 17) |
           ((kM / 16u) << 24);
}

// shared-memory matrix descriptor, 128-byte swizzle (sm_100 version bits)
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3fff) | ((uint64_t)((lbo >> 4) & 0x3fff) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3fff) << 32) | (1ull << 46) | (2ull << 61);
}

// The MMA and commit helpers are called by a whole warp with warp-uniform operands;
// elect.sync picks the one lane that issues (the operands stay warp-uniform, which
// keeps the issue cost per MMA low).
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t id,
                                       uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred e, p;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(id), "r"(acc));
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t id,
                                       uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred e, p;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(id), "r"(acc));
}
__device__ __forceinline__ void commit(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
            ptx::smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t addr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(addr));
}
__device__ __forceinline__ void tmem_st32(uint32_t addr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(addr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
        "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 2^x with the MUFU instruction (ftz; relative error ~2^-22, far inside what the
// bf16 weights keep); ex2(-inf) = 0
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// bounded wait; false (and the abort flag set) on timeout
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, int *abort_flag) {
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (*(volatile int *)abort_flag) return false;
        if (ptx::globaltimer() - t0 > kWaitNs) {
            atomicExch(abort_flag, 1);
            return false;
        }
    }
    return true;
}

// the same wait for every lane of a warp, with one warp-wide verdict (the
// tcgen05.ld/st that follow are warp-collective)
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int *abort_flag) {
    return __all_sync(0xffffffffu, wait_bar(bar, parity, abort_flag));
}

struct Bars {
    uint64_t q_full;              // 256 softmax threads: Q rows in shared memory
    uint64_t kv_full[kStages];    // TMA bytes of a K/V stage
    uint64_t kv_empty[kStages];   // commit after the last P V that read the stage
    uint64_t s_full[2];           // per Q tile: commit after S = Q K^T
    uint64_t p_full[2];           // per Q tile: 128 softmax threads wrote P
    uint64_t pv_done[2];          // per Q tile: commit after O += P V
    uint64_t o_final;             // commit after the last P V of both tiles
    uint32_t tmem_base;
    int abort_flag;
};

__global__ void __launch_bounds__(kThreads, 1)
    prefill_attn_tc_kernel(const __grid_constant__ CUtensorMap km,
                           const __grid_constant__ CUtensorMap vm, const PrefillAttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ Bars bars;
    const int b = blockIdx.z, h = blockIdx.y;
    const int G = a.G, QT = kRows / G;   // query tokens per CTA (two tiles of 128 rows)
    const int q0 = a.cu_q[b], ql = a.cu_q[b + 1] - q0;
    const int n_qt = (ql + QT - 1) / QT;
    const int qt = n_qt - 1 - (int)blockIdx.x;   // longest context first
    if (qt < 0) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int len = a.ctx_lens[b];
    const int tok_base = qt * QT;
    if (len < 0 || (int64_t)len > (int64_t)a.MB * a.bs || ql > len) {
        if (blockIdx.x == 0 && h == 0 && tid == 0) raise_flag(a.err, PA_DEV_BAD_LEN);
        for (int r = warp; r < kRows; r += kThreads / 32) {
            const int i = tok_base + r / G;
            if (i >= ql) continue;
            uint16_t *o = a.out + ((int64_t)(q0 + i) * a.Hq + h * G + r % G) * kD;
            for (int e = lane; e < kD; e += 32) o[e] = 0;
        }
        return;
    }
    const int pos0 = len - ql;
    const int last_tok = min(ql - 1, tok_base + QT - 1);
    const int p_max = pos0 + last_tok;
    const int n_kt = p_max / kN + 1;

    // 1024-byte aligned tiles (the 128-byte swizzle pattern repeats every 1024 bytes)
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    auto sQ = [&](int w) { return base + (uint32_t)(w * kTileB); };
    auto sK = [&](int st) { return base + (uint32_t)(2 * kTileB + st * 2 * kTileB); };
    auto sV = [&](int st) { return base + (uint32_t)(3 * kTileB + st * 2 * kTileB); };

    // K/V stages start as zeros: a page that is not loaded (bad block id) then
    // holds finite data only
    for (int x = tid; x < kStages * 2 * kTileB / 16; x += kThreads)
        *reinterpret_cast<uint4 *>(gbase + 2 * kTileB + 16 * x) = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (tid == 0) {
        ptx::mbar_init(&bars.q_full, 256);
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(&bars.kv_full[i], 1);
            ptx::mbar_init(&bars.kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&bars.s_full[i], 1);
            ptx::mbar_init(&bars.p_full[i], 128);
            ptx::mbar_init(&bars.pv_done[i], 1);
        }
        ptx::mbar_init(&bars.o_final, 1);
        bars.abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         ptx::smem_u32(&bars.tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tm = bars.tmem_base;
    int *abort_flag = &bars.abort_flag;

    if (warp < 8) {
        // ======================= softmax: warpgroup w owns Q tile w =======================
        const int w = warp >> 2;
        const int r = tid & 127;                 // row of the tile = TMEM lane
        const int R = w * 128 + r;               // row of the CTA
        const int i = tok_base + R / G;          // query token in the sequence's chunk
        const bool valid = i < ql;
        const int pos = pos0 + min(i, ql - 1);   // causal limit (inclusive)
        {   // Q row -> shared memory, K-major 128-byte swizzle
            const uint4 *src = reinterpret_cast<const uint4 *>(
                a.q + ((int64_t)(q0 + min(i, ql - 1)) * a.Hq + h * G + R % G) * kD);
            uint8_t *q = gbase + w * kTileB;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const uint4 v = src[c];
                const uint32_t off =
                    (uint32_t)((c >> 3) * kSlice + r * 128 + (((c & 7) ^ (r & 7)) << 4));
                *reinterpret_cast<uint4 *>(q + off) = v;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            ptx::mbar_arrive(&bars.q_full);
        }
        const uint32_t lane_base = tm + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t sbuf = lane_base + w * 128;          // S, then P over it
        const uint32_t obuf = lane_base + kColO + w * 128;  // O
        const float sl = a.scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_kt && ok; ++j) {
            if (!(ok = warp_wait(&bars.s_full[w], j & 1, abort_flag))) break;
            fence_after();
            // tokens t0 + e with e <= lim are visible to this row (lim >= 127: all)
            const int lim = valid ? pos - j * kN : -1;
            // tiles every row of the warp sees in full (all but the diagonal ones) skip
            // the causal select; with scale > 0 the max is taken on the raw logits
            const bool full = __all_sync(0xffffffffu, lim >= kN - 1) && sl > 0.f;
            // ---- the row's 128 logits of this tile: four 32-column TMEM reads in
            // flight, one wait; then the row maximum of the scaled, masked logits (8
            // independent max chains)
            uint32_t v[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(sbuf + 32 * c, v[c]);
            tmem_wait_ld();
            float mk[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) mk[q] = -INFINITY;
            if (full) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        mk[e & 7] = fmaxf(mk[e & 7], __uint_as_float(v[c][e]));
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float x =
                            (32 * c + e <= lim) ? __uint_as_float(v[c][e]) * sl : -INFINITY;
                        mk[e & 7] = fmaxf(mk[e & 7], x);
                    }
            }
            float mx = fmaxf(fmaxf(fmaxf(mk[0], mk[1]), fmaxf(mk[2], mk[3])),
                             fmaxf(fmaxf(mk[4], mk[5]), fmaxf(mk[6], mk[7])));
            if (full) mx *= sl;
            const float mn = fmaxf(m, mx);
            // lazy rescale: a row moves its reference max only when the tile's max
            // exceeds it by more than 8 (weights stay below 2^8 otherwise); the first
            // finite max always moves it (-inf + 8 = -inf)
            const bool move = mn > m + 8.f;
            const bool rescale = move && j > 0 && m != -INFINITY;  // O holds tiles < j
            const float alpha = rescale ? ex2(m - mn) : 1.f;
            if (move) m = mn;
            const float u = m == -INFINITY ? 0.f : m;
            // ---- pass 2: P = exp2(s - u) as hi + lo bf16 over the S columns: k-step kk
            // (16 tokens) at columns 16kk (hi, 8 columns of bf16 pairs) and 16kk + 8 (lo)
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float x[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = fmaf(__uint_as_float(v[c][e]), sl, -u);
                if (!full) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (32 * c + e > lim) x[e] = -INFINITY;  // weight 0
                }
                uint32_t wv[32];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int e = 16 * half + 2 * q;
                        const float p0 = ex2(x[e]), p1 = ex2(x[e + 1]);
                        ls[q & 3] += p0 + p1;
                        const uint32_t hi = ptx::pack_bf16(p0, p1);
                        wv[16 * half + q] = hi;
                        wv[16 * half + 8 + q] = ptx::pack_bf16(p0 - bf16_lo(hi), p1 - bf16_hi(hi));
                    }
                }
                tmem_st32(sbuf + 32 * c, wv);
            }
            // O is rescaled after P is written, when the logits' registers are free; the
            // P V of this tile is issued only after the arrive below
            if (__any_sync(0xffffffffu, rescale)) {   // warp-collective TMEM access
                if (!(ok = warp_wait(&bars.pv_done[w], (j - 1) & 1, abort_flag))) break;
                fence_after();
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tmem_ld32(obuf + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(obuf + 32 * c, o);
                }
            }
            l = l * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
            tmem_wait_st();
            fence_before();
            ptx::mbar_arrive(&bars.p_full[w]);
        }
        if (ok && warp_wait(&bars.o_final, 0, abort_flag)) {
            fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            uint4 *orow = reinterpret_cast<uint4 *>(
                a.out + ((int64_t)(q0 + min(i, ql - 1)) * a.Hq + h * G + R % G) * kD);
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
                tmem_ld32(obuf + 32 * c, v);
                tmem_wait_ld();
                if (valid) {   // 32 dims = 64 bytes of the row, as four 16-byte stores
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        uint32_t w4[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int e = 4 * e4 + k;
                            w4[k] = (uint32_t)f32_to_bf16_rn(__uint_as_float(v[2 * e]) * inv) |
                                    ((uint32_t)f32_to_bf16_rn(__uint_as_float(v[2 * e + 1]) * inv)
                                     << 16);
                        }
                        orow[4 * c + e4] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
            }
        }
    } else if (warp == 8) {
        // ======================= MMA issue =======================
        // tensor-core order per K/V tile j: PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so
        // each softmax warpgroup works while the other tile's products run
        const uint32_t id_qk = idesc(false), id_pv = idesc(true);
        auto zero_tail = [&](int j, int st) {
            // V rows at or past the context end: zero them (the weights there are 0,
            // and 0 x NaN would still poison the sum)
            const int t0 = j * kN;
            if (t0 + kN <= len) return;
            const int r0 = max(0, len - t0);
            for (int x = r0 * 16 + lane; x < kN * 16; x += 32) {
                const int row = x >> 4, c = x & 15;
                const uint32_t off = (uint32_t)((c >> 3) * kSlice + row * 128 + (c & 7) * 16);
                *reinterpret_cast<uint4 *>(gbase + (sV(st) - base) + off) = make_uint4(0, 0, 0, 0);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
        };
        auto issue_s = [&](int w, int st) {
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
                const uint32_t koff = (uint32_t)((ks >> 2) * kSlice + (ks & 3) * 32);
                mma_ss(tm + w * 128, sdesc(sQ(w) + koff, 16, 1024),
                       sdesc(sK(st) + koff, 16, 1024), id_qk, ks > 0);
            }
            commit(&bars.s_full[w]);
        };
        auto issue_pv = [&](int w, int j, int st) {
#pragma unroll
            for (int kk = 0; kk < kN / 16; ++kk) {
                // V: 16 token rows per k-step; N = 128 dims across the two slices
                const uint64_t vd = sdesc(sV(st) + (uint32_t)(kk * 16 * 128), kSlice, 1024);
                mma_ts(tm + kColO + w * 128, tm + w * 128 + 16 * kk, vd, id_pv,
                       (j > 0 || kk > 0) ? 1u : 0u);
                mma_ts(tm + kColO + w * 128, tm + w * 128 + 16 * kk + 8, vd, id_pv, 1u);
            }
            commit(&bars.pv_done[w]);
        };
        bool ok = warp_wait(&bars.q_full, 0, abort_flag) &&
                  warp_wait(&bars.kv_full[0], 0, abort_flag);
        if (ok) {
            zero_tail(0, 0);
            fence_after();
            issue_s(0, 0);
            issue_s(1, 0);
        }
        for (int j = 0; j < n_kt && ok; ++j) {
            const int st = j % kStages, st1 = (j + 1) % kStages;
            const bool more = j + 1 < n_kt;
            // ---- tile A
            if (!(ok = warp_wait(&bars.p_full[0], j & 1, abort_flag))) break;
            fence_after();
            issue_pv(0, j, st);
            if (more) {
                if (!(ok = warp_wait(&bars.kv_full[st1], ((j + 1) / kStages) & 1, abort_flag))) break;
                zero_tail(j + 1, st1);
                // S_A(j+1) overwrites the columns PV_A(j) reads its P from
                if (!(ok = warp_wait(&bars.pv_done[0], j & 1, abort_flag))) break;
                fence_after();
                issue_s(0, st1);
            }
            // ---- tile B
            if (!(ok = warp_wait(&bars.p_full[1], j & 1, abort_flag))) break;
            fence_after();
            issue_pv(1, j, st);
            commit(&bars.kv_empty[st]);
            if (!more) commit(&bars.o_final);
            if (more) {
                if (!(ok = warp_wait(&bars.pv_done[1], j & 1, abort_flag))) break;
                fence_after();
                issue_s(1, st1);
            }
        }
    } else {
        // ======================= TMA producer (warp 9) =======================
        // lane pg < 8 owns 16-token page pg of every tile: it looks up the page's
        // physical block (one tile ahead, so the table read is off the critical
        // path) and issues the page's four boxes
        const int32_t *btr = a.block_tables + (int64_t)b * a.MB;
        auto lookup = [&](int j) -> int32_t {
            const int t = j * kN + 16 * lane;
            return (lane < kN / 16 && t < len) ? btr[t / a.bs] : -1;
        };
        int32_t next = lookup(0);
        bool ok = true;
        for (int j = 0; j < n_kt && ok; ++j) {
            const int st = j % kStages;
            const int32_t blk = next;
            if (j + 1 < n_kt) next = lookup(j + 1);
            if (j >= kStages &&
                !(ok = warp_wait(&bars.kv_empty[st], ((j / kStages) - 1) & 1, abort_flag)))
                break;
            const int t = j * kN + 16 * lane;
            const bool in = lane < kN / 16 && t < len;
            // pages inside the context with a valid block id are loaded; the others
            // are not (their rows are masked, and V rows past the end zeroed)
            const bool load = in && blk >= 0 && (int64_t)blk < a.N;
            if (in && !load) raise_flag(a.err, PA_DEV_BAD_BLOCK);
            const unsigned lm = __ballot_sync(0xffffffffu, load);
            if (lane == 0)
                ptx::mbar_arrive_expect_tx(&bars.kv_full[st], (uint32_t)__popc(lm) * 4u * 2048u);
            __syncwarp();
            if (load) {
                const int off = t % a.bs;
#pragma unroll
                for (int sl = 0; sl < 2; ++sl) {
                    const uint32_t dk = sK(st) + (uint32_t)(sl * kSlice + lane * 16 * 128);
                    const uint32_t dv = sV(st) + (uint32_t)(sl * kSlice + lane * 16 * 128);
                    ptx::tma_load_5d(gbase + (dk - base), &km, &bars.kv_full[st], 0, off, h, sl,
                                     blk);
                    ptx::tma_load_5d(gbase + (dv - base), &vm, &bars.kv_full[st], 0, off, h, sl,
                                     blk);
                }
            }
        }
    }
    if (*(volatile int *)abort_flag && tid == 0) raise_flag(a.err, PA_DEV_TIMEOUT);
    fence_before();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm),
                     "r"(kTmemCols));
}

PFN_cuTensorMapEncodeTiled_v12000 tc_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [blocks][bs][Hkv][2 slices][64] view of a bf16 pool; box = 16 tokens of one head
// and one 64-element slice (2 KB), 128-byte swizzle
bool encode_head_map(CUtensorMap *map, const void *base, int64_t N, int bs, int Hkv,
                     int64_t block_stride) {
    auto fn = tc_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[5] = {64, (cuuint64_t)bs, (cuuint64_t)Hkv, 2, (cuuint64_t)N};
    const cuuint64_t strides[4] = {(cuuint64_t)Hkv * kD * 2, (cuuint64_t)kD * 2, 128,
                                   (cuuint64_t)block_stride * 2};
    const cuuint32_t box[5] = {64, 16, 1, 1, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 5, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool prefill_attn_tc_supported(const PrefillAttnArgs &a) {
    return a.d == kD && a.bs % 16 == 0;
}

cudaError_t launch_prefill_attn_tc(const PrefillAttnArgs &a, int max_q_len, cudaStream_t st) {
    CUtensorMap km, vm;
    if (!encode_head_map(&km, a.k_cache, a.N, a.bs, a.Hkv, a.block_stride) ||
        !encode_head_map(&vm, a.v_cache, a.N, a.bs, a.Hkv, a.block_stride))
        return cudaErrorInvalidValue;
    static bool attr_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    if (dev >= 64 || !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(prefill_attn_tc_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set[dev] = true;
    }
    const int QT = kRows / a.G;
    dim3 grid((unsigned)((max_q_len + QT - 1) / QT), (unsigned)a.Hkv, (unsigned)a.B);
    prefill_attn_tc_kernel<<<grid, kThreads, kSmem, st>>>(km, vm, a);
    return cudaGetLastError();
}

}  // namespace pkv
