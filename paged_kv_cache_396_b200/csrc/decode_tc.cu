// decode_tc.cu -- paged decode attention for block sizes that are a multiple of
// 16: TMA-staged K/V tiles, bf16 tensor-core QK^T and PV, online softmax.
//
// Operator (ybb.press "LLM 推理 KV Cache 内存管理深度工程实践" §2.2 paged_attention_forward;
// t6page.pages.dev "KV cache", "PagedAttention 的算子"): for each sequence the K/V
// rows are found through the block table, and softmax(scale q.K) V is taken over
// the whole context; GQA (§6.2 of the first page): query head i reads kv head i/G.
//
// Work decomposition
//   A plan kernel (one CTA) reads the device context lengths, cuts every
//   sequence into near-equal partitions of at most `chunk` tokens (chunk sized
//   so that there are a few partitions per SM), and writes the partitions as a
//   unit list sorted longest first.  The decode kernel is persistent (one CTA
//   per SM); its producer warp takes units from an atomic counter, so long units
//   start first and short ones fill the tail.
// Per CTA
//   warp 8 (producer): for each stage of 16*n_sub tokens, looks the physical
//   blocks up in the block table and issues 5-D TMA loads of the K and V rows of
//   ALL kv heads of 16 consecutive tokens (one box per 64-element slice of d),
//   plus, on a unit's first stage, a bulk copy of the sequence's query rows.
//   The tensor map orders the box as [head][token][64 elements] with 128-byte
//   swizzle, so each head's 16 token rows occupy 16 consecutive 128-byte rows
//   and ldmatrix reads them without bank conflicts.
//   warps 0..7 (consumers): warp w owns kv head w % Hkv and 16-token sub-tile
//   w / Hkv of every stage.  S = Q K^T with the G query heads of the group as
//   the 16 rows of an m16n8k16 MMA (rows >= G are zero), online softmax on the
//   fp32 accumulators (exp2 domain), P rounded to bf16, O += P V with V read by
//   ldmatrix.trans.  The stage is released to the producer through an mbarrier.
//   At a unit's last stage the warp writes either the normalised bf16 output
//   (single-partition sequence) or its (O, m, l) partial for the merge kernel.
// Masking: tokens at or past the unit's end get -inf logits, and their V rows
// are zeroed in registers, so stale or NaN data in unused slots never reaches
// the result.  Out-of-range block ids are not loaded; the sub-tile is skipped
// and PA_DEV_BAD_BLOCK is raised.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace pkv {
namespace tc {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kTile = 16;
constexpr int kBoxRow = 128;  // bytes per (head, token) row of one box (64 bf16)
constexpr uint32_t kFull = 0xffffffffu;

enum : int { kFirst = 1, kLast = 2, kEnd = 4, kDirect = 8 };

struct StageMeta {
    int b, c, ts, te;  // sequence, partition, token range [ts, te) of this stage
    int flags;
    int bad;           // bit j: sub-tile j skipped (block id out of range)
    int pad[2];
};

struct Args {
    const uint16_t *q;
    uint16_t *out;
    const int32_t *bt;
    const int32_t *ctx_lens;
    int32_t *err;
    TcHeader *hdr;
    const int4 *units;
    const int32_t *ns;
    float *ws_acc;
    float *ws_ml;
    int64_t N;
    int B, Hq, Hkv, G, bs, MB, S, n_sub, nstage, stage_bytes, q_off, v_off, box_bytes;
    float scale_log2;
};

// ---------------------------------------------------------------------------
// plan: one CTA of 1024 threads
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t *ctx_lens, int32_t *err,
                                                   TcHeader *hdr, int32_t *ns, int4 *units, int B,
                                                   int max_ctx, int min_chunk, int target_units) {
    __shared__ long long s_red[32];
    __shared__ int hist[1024];
    __shared__ int s_chunk;
    const int tid = threadIdx.x;
    long long tot = 0;
    for (int b = tid; b < B; b += blockDim.x) {
        int len = ctx_lens[b];
        if (len < 0 || len > max_ctx) {
            raise_flag(err, PA_DEV_BAD_LEN);
            len = 0;
        }
        tot += len;
    }
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(kFull, tot, o);
    if ((tid & 31) == 0) s_red[tid >> 5] = tot;
    for (int i = tid; i < 1024; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    if (tid == 0) {
        long long t = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += s_red[w];
        long long ch = (t + target_units - 1) / target_units;
        ch = (ch + kTile - 1) / kTile * kTile;
        if (ch < min_chunk) ch = min_chunk;
        if (ch > max_ctx) ch = (max_ctx + kTile - 1) / kTile * kTile;
        s_chunk = (int)ch;
        hdr->chunk = (int)ch;
    }
    __syncthreads();
    const int chunk = s_chunk;
    // partitions: near-equal, 16-token aligned; bucket by size for longest-first order
    auto part = [&](int len, int &n, int &step) {
        n = len > 0 ? (len + chunk - 1) / chunk : 1;
        step = len > 0 ? ((len + n - 1) / n + kTile - 1) / kTile * kTile : kTile;
        n = len > 0 ? (len + step - 1) / step : 1;
    };
    for (int b = tid; b < B; b += blockDim.x) {
        int len = ctx_lens[b];
        if (len < 0 || len > max_ctx) len = 0;
        int n, step;
        part(len, n, step);
        ns[b] = n;
        for (int c = 0; c < n; ++c) {
            const int sz = min(step, len - c * step);
            atomicAdd(&hist[min(1023, sz / kTile)], 1);
        }
    }
    __syncthreads();
    if (tid == 0) {  // exclusive prefix, largest bucket first
        int run = 0;
        for (int k = 1023; k >= 0; --k) {
            const int c = hist[k];
            hist[k] = run;
            run += c;
        }
        hdr->n_units = run;
        hdr->counter = 0u;
    }
    __syncthreads();
    for (int b = tid; b < B; b += blockDim.x) {
        int len = ctx_lens[b];
        if (len < 0 || len > max_ctx) len = 0;
        int n, step;
        part(len, n, step);
        for (int c = 0; c < n; ++c) {
            const int t0 = c * step, t1 = min(len, t0 + step);
            const int pos = atomicAdd(&hist[min(1023, (t1 - t0) / kTile)], 1);
            units[pos] = make_int4(b, c, t0, t1);
        }
    }
}

// ---------------------------------------------------------------------------
// decode: persistent, warp-specialised
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void producer(const CUtensorMap *kmap, const CUtensorMap *vmap,
                                         const Args &a, uint8_t *stages, StageMeta *meta,
                                         uint64_t *full, uint64_t *empty) {
    constexpr int DC = D / 64;
    const int lane = threadIdx.x & 31;
    const int T_s = kTile * a.n_sub;
    const uint32_t qbytes = (uint32_t)a.Hq * D * 2;
    const int n_units = a.hdr->n_units;
    const uint64_t policy = ptx::policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    if (lane == 0) {
        ptx::prefetch_tensormap(kmap);
        ptx::prefetch_tensormap(vmap);
    }
    while (ok) {
        unsigned u = 0;
        if (lane == 0) u = atomicAdd(&a.hdr->counter, 1u);
        u = __shfl_sync(kFull, u, 0);
        if ((int)u >= n_units) break;
        const int4 un = a.units[u];
        const int b = un.x, c = un.y, t0 = un.z, t1 = un.w;
        const bool direct = (a.n_sub == 1) && (a.ns[b] == 1);
        const int nst = t1 > t0 ? (t1 - t0 + T_s - 1) / T_s : 1;
        const int32_t *bt_row = a.bt + (int64_t)b * a.MB;
        int cache_base = -1, cache = 0;  // lane k caches the id of block cache_base + k
        for (int si = 0; si < nst; ++si) {
            const int ts = t0 + si * T_s, te = min(ts + T_s, t1);
            if (te > ts) {
                const int last_blk = (te - 1) / a.bs;
                if (cache_base < 0 || last_blk >= cache_base + 32) {
                    cache_base = ts / a.bs;
                    const int blk = cache_base + lane;
                    cache = blk <= (t1 - 1) / a.bs ? __ldg(bt_row + blk) : -1;
                }
            }
            int phys[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int tok = ts + kTile * j;
                const int idx = (j < a.n_sub && tok < te) ? tok / a.bs - cache_base : 0;
                phys[j] = __shfl_sync(kFull, cache, idx & 31);
            }
            if (!ptx::mbar_wait(&empty[stage], phase ^ 1u)) {
                if (lane == 0) raise_flag(a.err, PA_DEV_TIMEOUT);
                ok = false;
                break;
            }
            if (lane == 0) {
                uint8_t *sb = stages + (size_t)stage * a.stage_bytes;
                uint32_t bytes = 0;
                int bad = 0;
                for (int j = 0; j < a.n_sub; ++j) {
                    const int tok = ts + kTile * j;
                    if (tok >= te) break;
                    if (phys[j] < 0 || (int64_t)phys[j] >= a.N) {
                        bad |= 1 << j;
                        continue;
                    }
                    bytes += 2u * DC * (uint32_t)a.box_bytes;
                }
                if (si == 0) bytes += qbytes;
                StageMeta &m = meta[stage];
                m.b = b;
                m.c = c;
                m.ts = ts;
                m.te = te;
                m.bad = bad;
                m.flags = (si == 0 ? kFirst : 0) | (si == nst - 1 ? kLast : 0) |
                          (direct ? kDirect : 0);
                if (bad) raise_flag(a.err, PA_DEV_BAD_BLOCK);
                ptx::mbar_arrive_expect_tx(&full[stage], bytes);
                for (int j = 0; j < a.n_sub; ++j) {
                    const int tok = ts + kTile * j;
                    if (tok >= te) break;
                    if ((bad >> j) & 1) continue;
                    const int slot = tok % a.bs;
#pragma unroll
                    for (int dc = 0; dc < DC; ++dc) {
                        const size_t off = (size_t)(j * DC + dc) * a.box_bytes;
                        ptx::tma_load_5d_hint(sb + off, kmap, &full[stage], 0, slot, 0, dc, phys[j],
                                              policy);
                        ptx::tma_load_5d_hint(sb + a.v_off + off, vmap, &full[stage], 0, slot, 0,
                                              dc, phys[j], policy);
                    }
                }
                if (si == 0) ptx::bulk_load(sb + a.q_off, a.q + (int64_t)b * a.Hq * D, qbytes,
                                            &full[stage]);
            }
            __syncwarp();
            if (++stage == a.nstage) {
                stage = 0;
                phase ^= 1u;
            }
        }
    }
    if (ok) {
        if (ptx::mbar_wait(&empty[stage], phase ^ 1u)) {
            if (lane == 0) {
                meta[stage].flags = kEnd;
                ptx::mbar_arrive(&full[stage]);
            }
        } else if (lane == 0) {
            raise_flag(a.err, PA_DEV_TIMEOUT);
        }
    }
}

template <int D, bool G16>
__device__ __forceinline__ void consumer(const Args &a, uint8_t *stages, StageMeta *meta,
                                         uint64_t *full, uint64_t *empty) {
    constexpr int DC = D / 64;
    constexpr int KS = D / 16;  // k-steps of QK^T (and n-tile pairs of PV)
    constexpr int NT = D / 8;   // n-tiles of the output
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = warp % a.Hkv, j = warp / a.Hkv;
    const int g = lane >> 2, tig = lane & 3;
    const int mi = lane >> 3, ri = lane & 7;
    // per-lane byte offsets inside a (head, sub-tile, 64-element) box
    const int tk = ri + ((mi >> 1) << 3);        // K: matrices 0,1 -> tokens 0-7; 2,3 -> 8-15
    const int ck = mi & 1;                       //    matrices 1,3 -> second 16-byte chunk
    const int tv = ri + ((mi & 1) << 3);         // V: matrices 0,2 -> tokens 0-7; 1,3 -> 8-15
    const int cv = mi >> 1;
    const uint32_t stage0 = ptx::smem_u32(stages);
    const uint32_t head_off = (uint32_t)(j * DC * a.box_bytes + h * kTile * kBoxRow);

    uint32_t qa[KS][2];
    uint32_t qb[G16 ? KS : 1][2];
    float o[NT][2];
    float ob[G16 ? NT : 1][2];
    float m = -INFINITY, l = 0.f, mb = -INFINITY, lb = 0.f;
    int stage = 0;
    uint32_t phase = 0;
    for (;;) {
        if (!ptx::mbar_wait(&full[stage], phase)) {
            if (lane == 0) raise_flag(a.err, PA_DEV_TIMEOUT);
            break;
        }
        const StageMeta mt = meta[stage];
        if (mt.flags & kEnd) break;
        const uint32_t sb = stage0 + (uint32_t)stage * a.stage_bytes;
        if (mt.flags & kFirst) {
            const uint32_t qs = sb + a.q_off;
            const int row = h * a.G + g;
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                const uint32_t ad = qs + (uint32_t)((row * D + kk * 16 + 2 * tig) * 2);
                qa[kk][0] = g < a.G ? ptx::lds32(ad) : 0u;
                qa[kk][1] = g < a.G ? ptx::lds32(ad + 16) : 0u;
                if constexpr (G16) {
                    const uint32_t adb = ad + 8 * D * 2;
                    qb[kk][0] = g + 8 < a.G ? ptx::lds32(adb) : 0u;
                    qb[kk][1] = g + 8 < a.G ? ptx::lds32(adb + 16) : 0u;
                }
            }
            m = -INFINITY;
            l = 0.f;
            mb = -INFINITY;
            lb = 0.f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                o[nt][0] = o[nt][1] = 0.f;
                if constexpr (G16) ob[nt][0] = ob[nt][1] = 0.f;
            }
        }
        const int tj = mt.ts + kTile * j;
        const int nv = max(0, min(kTile, mt.te - tj));
        if (nv > 0 && !((mt.bad >> j) & 1)) {
            const uint32_t kbase = sb + head_off;
            const uint32_t vbase = sb + a.v_off + head_off;
            // ---- S = Q K^T : two n-tiles of 8 tokens
            float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                const int dc = kk >> 2, c = ((kk & 3) << 1) + ck;
                uint32_t r[4];
                ptx::ldmatrix_x4(r, kbase + dc * a.box_bytes + tk * kBoxRow + ((c ^ ri) << 4));
                if constexpr (G16) {
                    ptx::mma_bf16(s0, qa[kk][0], qb[kk][0], qa[kk][1], qb[kk][1], r[0], r[1]);
                    ptx::mma_bf16(s1, qa[kk][0], qb[kk][0], qa[kk][1], qb[kk][1], r[2], r[3]);
                } else {
                    ptx::mma_bf16(s0, qa[kk][0], 0u, qa[kk][1], 0u, r[0], r[1]);
                    ptx::mma_bf16(s1, qa[kk][0], 0u, qa[kk][1], 0u, r[2], r[3]);
                }
            }
            // ---- online softmax (rows g and, for G > 8, g + 8)
            const int t_a = 2 * tig, t_b = 8 + 2 * tig;
            const bool va0 = t_a < nv, va1 = t_a + 1 < nv, vb0 = t_b < nv, vb1 = t_b + 1 < nv;
            const float sl = a.scale_log2;
            float x0 = va0 ? s0[0] * sl : -INFINITY, x1 = va1 ? s0[1] * sl : -INFINITY;
            float x2 = vb0 ? s1[0] * sl : -INFINITY, x3 = vb1 ? s1[1] * sl : -INFINITY;
            float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
            const float mn = fmaxf(m, mx);
            const float mu = mn == -INFINITY ? 0.f : mn;
            const float alpha = exp2f(m - mu);
            const float p0 = exp2f(x0 - mu), p1 = exp2f(x1 - mu);
            const float p2 = exp2f(x2 - mu), p3 = exp2f(x3 - mu);
            l = l * alpha + ((p0 + p1) + (p2 + p3));
            m = mn;
            const uint32_t pa0 = ptx::pack_bf16(p0, p1), pa2 = ptx::pack_bf16(p2, p3);
            uint32_t pa1 = 0u, pa3 = 0u;
            float alphab = 1.f;
            if constexpr (G16) {
                float y0 = va0 ? s0[2] * sl : -INFINITY, y1 = va1 ? s0[3] * sl : -INFINITY;
                float y2 = vb0 ? s1[2] * sl : -INFINITY, y3 = vb1 ? s1[3] * sl : -INFINITY;
                float my = fmaxf(fmaxf(y0, y1), fmaxf(y2, y3));
                my = fmaxf(my, __shfl_xor_sync(kFull, my, 1));
                my = fmaxf(my, __shfl_xor_sync(kFull, my, 2));
                const float mnb = fmaxf(mb, my);
                const float mub = mnb == -INFINITY ? 0.f : mnb;
                alphab = exp2f(mb - mub);
                const float q0 = exp2f(y0 - mub), q1 = exp2f(y1 - mub);
                const float q2 = exp2f(y2 - mub), q3 = exp2f(y3 - mub);
                lb = lb * alphab + ((q0 + q1) + (q2 + q3));
                mb = mnb;
                pa1 = ptx::pack_bf16(q0, q1);
                pa3 = ptx::pack_bf16(q2, q3);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                o[nt][0] *= alpha;
                o[nt][1] *= alpha;
                if constexpr (G16) {
                    ob[nt][0] *= alphab;
                    ob[nt][1] *= alphab;
                }
            }
            // ---- O += P V
            const uint32_t mlo = (va0 ? 0x0000ffffu : 0u) | (va1 ? 0xffff0000u : 0u);
            const uint32_t mhi = (vb0 ? 0x0000ffffu : 0u) | (vb1 ? 0xffff0000u : 0u);
            const bool partial = nv < kTile;
#pragma unroll
            for (int jj = 0; jj < KS; ++jj) {
                const int dc = jj >> 2, c = ((jj & 3) << 1) + cv;
                uint32_t r[4];
                ptx::ldmatrix_x4_trans(r, vbase + dc * a.box_bytes + tv * kBoxRow +
                                              ((c ^ ri) << 4));
                if (partial) {
                    r[0] &= mlo;
                    r[1] &= mhi;
                    r[2] &= mlo;
                    r[3] &= mhi;
                }
                float d0[4] = {o[2 * jj][0], o[2 * jj][1], 0.f, 0.f};
                float d1[4] = {o[2 * jj + 1][0], o[2 * jj + 1][1], 0.f, 0.f};
                if constexpr (G16) {
                    d0[2] = ob[2 * jj][0];
                    d0[3] = ob[2 * jj][1];
                    d1[2] = ob[2 * jj + 1][0];
                    d1[3] = ob[2 * jj + 1][1];
                }
                ptx::mma_bf16(d0, pa0, pa1, pa2, pa3, r[0], r[1]);
                ptx::mma_bf16(d1, pa0, pa1, pa2, pa3, r[2], r[3]);
                o[2 * jj][0] = d0[0];
                o[2 * jj][1] = d0[1];
                o[2 * jj + 1][0] = d1[0];
                o[2 * jj + 1][1] = d1[1];
                if constexpr (G16) {
                    ob[2 * jj][0] = d0[2];
                    ob[2 * jj][1] = d0[3];
                    ob[2 * jj + 1][0] = d1[2];
                    ob[2 * jj + 1][1] = d1[3];
                }
            }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[stage]);
        if (mt.flags & kLast) {
            float lt = l + __shfl_xor_sync(kFull, l, 1);
            lt += __shfl_xor_sync(kFull, lt, 2);
            float ltb = 0.f;
            if constexpr (G16) {
                ltb = lb + __shfl_xor_sync(kFull, lb, 1);
                ltb += __shfl_xor_sync(kFull, ltb, 2);
            }
            const int row = h * a.G + g;
            if (mt.flags & kDirect) {
                if (g < a.G) {
                    const float inv = lt > 0.f ? 1.f / lt : 0.f;
                    uint32_t *dst = reinterpret_cast<uint32_t *>(
                        a.out + ((int64_t)mt.b * a.Hq + row) * D + 2 * tig);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        dst[nt * 4] = ptx::pack_bf16(o[nt][0] * inv, o[nt][1] * inv);
                }
                if constexpr (G16) {
                    if (g + 8 < a.G) {
                        const float inv = ltb > 0.f ? 1.f / ltb : 0.f;
                        uint32_t *dst = reinterpret_cast<uint32_t *>(
                            a.out + ((int64_t)mt.b * a.Hq + row + 8) * D + 2 * tig);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            dst[nt * 4] = ptx::pack_bf16(ob[nt][0] * inv, ob[nt][1] * inv);
                    }
                }
            } else {
                const int64_t slot = ((int64_t)mt.b * a.S + mt.c) * a.n_sub + j;
                if (g < a.G) {
                    const int64_t r = slot * a.Hq + row;
                    float2 *dst = reinterpret_cast<float2 *>(a.ws_acc + r * D + 2 * tig);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) dst[nt * 4] = make_float2(o[nt][0], o[nt][1]);
                    if (tig == 0) *reinterpret_cast<float2 *>(a.ws_ml + r * 2) = make_float2(m, lt);
                }
                if constexpr (G16) {
                    if (g + 8 < a.G) {
                        const int64_t r = slot * a.Hq + row + 8;
                        float2 *dst = reinterpret_cast<float2 *>(a.ws_acc + r * D + 2 * tig);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            dst[nt * 4] = make_float2(ob[nt][0], ob[nt][1]);
                        if (tig == 0)
                            *reinterpret_cast<float2 *>(a.ws_ml + r * 2) = make_float2(mb, ltb);
                    }
                }
            }
        }
        if (++stage == a.nstage) {
            stage = 0;
            phase ^= 1u;
        }
    }
}

template <int D, bool G16>
__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap, const Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *stages = smem;
    StageMeta *meta = reinterpret_cast<StageMeta *>(smem + (size_t)a.nstage * a.stage_bytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(meta + a.nstage);
    uint64_t *empty = full + a.nstage;
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.nstage; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], kConsumerWarps);
        }
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if ((threadIdx.x >> 5) == kConsumerWarps)
        producer<D>(&kmap, &vmap, a, stages, meta, full, empty);
    else
        consumer<D, G16>(a, stages, meta, full, empty);
}

// Merge of the partials of one (sequence, query head) in slot order.
template <int D>
__global__ void __launch_bounds__(D) merge_tc_kernel(const Args a) {
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / a.Hq), i = (int)(bh % a.Hq);
    const int e = threadIdx.x;
    const int nsb = a.ns[b];
    if (nsb == 1 && a.n_sub == 1) return;  // written directly by the decode kernel
    const int cnt = nsb * a.n_sub;
    const int64_t base = (int64_t)b * a.S * a.n_sub;
    float M = -INFINITY;
    for (int s = 0; s < cnt; ++s) M = fmaxf(M, a.ws_ml[((base + s) * a.Hq + i) * 2]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < cnt; ++s) {
            const int64_t r = (base + s) * a.Hq + i;
            const float f = exp2f(a.ws_ml[r * 2] - M);
            L = fmaf(a.ws_ml[r * 2 + 1], f, L);
            A = fmaf(a.ws_acc[r * D + e], f, A);
        }
    }
    a.out[bh * D + e] = f32_to_bf16_rn(L > 0.f ? A / L : 0.f);
}

// ---------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// Pool viewed as 5-D (innermost first): 64 elements of d | slot in block |
// kv head | 64-element slice of d | physical block.  Box (64, 16, Hkv, 1, 1):
// in shared memory [head][token][64 elements], 128-byte swizzled.
bool encode_pool_map(CUtensorMap *map, const void *base, int64_t N, int bs, int Hkv, int d,
                     int64_t block_stride) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[5] = {64, (cuuint64_t)bs, (cuuint64_t)Hkv, (cuuint64_t)(d / 64),
                                (cuuint64_t)N};
    const cuuint64_t strides[4] = {(cuuint64_t)Hkv * d * 2, (cuuint64_t)d * 2, 128,
                                   (cuuint64_t)block_stride * 2};
    const cuuint32_t box[5] = {64, (cuuint32_t)kTile, (cuuint32_t)Hkv, 1, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D, bool G16>
cudaError_t launch_typed(const CUtensorMap &km, const CUtensorMap &vm, const Args &a, int grid,
                         int smem, cudaStream_t st) {
    auto kfn = decode_tc_kernel<D, G16>;
    static unsigned long long attr_set = 0;  // one bit per device; benign race (idempotent)
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !((attr_set >> dev) & 1ull)) {
        cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             227 * 1024);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set |= 1ull << dev;
    }
    kfn<<<grid, kThreads, smem, st>>>(km, vm, a);
    return cudaGetLastError();
}

}  // namespace tc

cudaError_t launch_decode_tc(const DecodeArgs &d, cudaStream_t st) {
    using namespace tc;
    const DecodePlan &p = d.plan;
    CUtensorMap km, vm;
    if (!encode_pool_map(&km, d.k_cache, d.N, d.bs, d.Hkv, d.d, d.block_stride) ||
        !encode_pool_map(&vm, d.v_cache, d.N, d.bs, d.Hkv, d.d, d.block_stride))
        return cudaErrorInvalidValue;
    char *ws = static_cast<char *>(d.ws);
    Args a;
    a.q = d.q;
    a.out = d.out;
    a.bt = d.block_tables;
    a.ctx_lens = d.ctx_lens;
    a.err = d.err;
    a.hdr = reinterpret_cast<TcHeader *>(ws + p.off_hdr);
    a.ns = reinterpret_cast<const int32_t *>(ws + p.off_ns);
    a.units = reinterpret_cast<const int4 *>(ws + p.off_units);
    a.ws_ml = reinterpret_cast<float *>(ws + p.off_ml);
    a.ws_acc = reinterpret_cast<float *>(ws + p.off_acc);
    a.N = d.N;
    a.B = d.B;
    a.Hq = d.Hq;
    a.Hkv = d.Hkv;
    a.G = d.G;
    a.bs = d.bs;
    a.MB = d.MB;
    a.S = p.S;
    a.n_sub = p.n_sub;
    a.nstage = p.nstage;
    a.stage_bytes = p.stage_bytes;
    a.q_off = p.q_off;
    a.v_off = p.v_off;
    a.box_bytes = d.Hkv * kTile * kBoxRow;
    a.scale_log2 = d.scale_log2;
    const int max_ctx = d.MB * d.bs;
    plan_kernel<<<1, 1024, 0, st>>>(d.ctx_lens, d.err, a.hdr, const_cast<int32_t *>(a.ns),
                                    const_cast<int4 *>(a.units), d.B, max_ctx, p.chunk,
                                    p.grid * p.units_per_cta);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const bool g16 = d.G > 8;
    if (d.d == 128)
        e = g16 ? launch_typed<128, true>(km, vm, a, p.grid, p.smem_bytes, st)
                : launch_typed<128, false>(km, vm, a, p.grid, p.smem_bytes, st);
    else
        e = g16 ? launch_typed<64, true>(km, vm, a, p.grid, p.smem_bytes, st)
                : launch_typed<64, false>(km, vm, a, p.grid, p.smem_bytes, st);
    if (e != cudaSuccess) return e;
    if (p.S > 1 || p.n_sub > 1) {
        const unsigned rows = (unsigned)((int64_t)d.B * d.Hq);
        if (d.d == 128) merge_tc_kernel<128><<<rows, 128, 0, st>>>(a);
        else merge_tc_kernel<64><<<rows, 64, 0, st>>>(a);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace pkv
