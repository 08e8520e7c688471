// decode_simple.cu -- paged decode attention, general-shape kernel, and the
// cross-partition log-sum-exp merge shared by every decode kernel.
//
// Operator (ybb.press "LLM 推理 KV Cache 内存管理深度工程实践" §2.2; t6page.pages.dev
// "KV cache", "PagedAttention 的算子"): for each sequence, K/V rows are found
// through the block table and softmax(scale * q.K) V is taken over the whole
// context.  GQA (§6.2 of the first page): query head i uses kv head i / G.
//
// This kernel handles any block size (one CTA per (partition, kv head,
// sequence), one warp per token, CUDA-core fp32).  Block sizes that are a
// multiple of 16 use the staged tensor-core kernel in decode_tc.cu instead.
// Softmax runs online in the log2 domain: logits are pre-scaled by
// scale*log2(e) so every exponential is an exp2.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace pkv {

// fp16 bits -> fp32 (exact)
__device__ __forceinline__ float half_bits_to_f32(uint16_t h) {
    float f;
    asm("{ .reg .f16 t; mov.b16 t, %1; cvt.f32.f16 %0, t; }" : "=f"(f) : "h"(h));
    return f;
}

// Two e4m3 codes (low byte first) -> two fp32, exactly (every e4m3 value is an fp16).
__device__ __forceinline__ void e4m3x2_to_f32(uint16_t c, float &lo, float &hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(c));
    lo = half_bits_to_f32((uint16_t)(r & 0xffffu));
    hi = half_bits_to_f32((uint16_t)(r >> 16));
}

template <int D, int KV>
__device__ __forceinline__ void load_kv_row(const void *base, int64_t idx, float (&x)[D / 32]) {
    constexpr int VEC = D / 32;
    if constexpr (KV == kKvInt8) {
        const int8_t *p = reinterpret_cast<const int8_t *>(base) + idx;
        if constexpr (VEC == 4) {
            const uint32_t w = __ldg(reinterpret_cast<const unsigned int *>(p));
#pragma unroll
            for (int e = 0; e < 4; ++e) x[e] = (float)(int8_t)((w >> (8 * e)) & 0xffu);
        } else {
            const uint16_t w = __ldg(reinterpret_cast<const unsigned short *>(p));
            x[0] = (float)(int8_t)(w & 0xffu);
            x[1] = (float)(int8_t)(w >> 8);
        }
    } else if constexpr (KV == kKvFp8) {
        const uint8_t *p = reinterpret_cast<const uint8_t *>(base) + idx;
        if constexpr (VEC == 4) {
            const uint32_t w = __ldg(reinterpret_cast<const unsigned int *>(p));
            e4m3x2_to_f32((uint16_t)(w & 0xffffu), x[0], x[1]);
            e4m3x2_to_f32((uint16_t)(w >> 16), x[2], x[3]);
        } else {
            e4m3x2_to_f32(__ldg(reinterpret_cast<const unsigned short *>(p)), x[0], x[1]);
        }
    } else {
        const uint16_t *p = reinterpret_cast<const uint16_t *>(base) + idx;
        if constexpr (VEC == 4) {
            const uint2 w = __ldg(reinterpret_cast<const uint2 *>(p));
            x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
        } else {
            const uint32_t w = __ldg(reinterpret_cast<const unsigned int *>(p));
            x[0] = bf16_lo(w); x[1] = bf16_hi(w);
        }
    }
}

// Grid (partition c, kv head h, sequence b); 4 warps; warp w takes tokens
// t0+w, t0+w+4, ... of the partition and keeps its own online-softmax state
// for the GP (>= G, power of two) query heads of the group; the four states are
// merged through shared memory at the end.
template <int D, int GP, int KV>
__global__ void __launch_bounds__(128) decode_simple_kernel(DecodeArgs a) {
    constexpr int VEC = D / 32;
    constexpr int NW = 4;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int len = a.ctx_lens[b];
    if (len < 0 || (int64_t)len > (int64_t)a.MB * a.bs) {
        if (c == 0 && h == 0 && threadIdx.x == 0) raise_flag(a.err, PA_DEV_BAD_LEN);
        len = 0;
    }
    const int t0 = c * a.chunk;
    if (c > 0 && t0 >= len) return;  // partition past the context: the merge skips it
    const int t1 = min(t0 + a.chunk, len);

    float qf[GP][VEC];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
        if (g < a.G) {
            float x[VEC];
            const int64_t qi = ((int64_t)b * a.Hq + h * a.G + g) * D + lane * VEC;
            load_kv_row<D, kKvBf16>(a.q, qi, x);
#pragma unroll
            for (int e = 0; e < VEC; ++e) qf[g][e] = x[e] * a.scale_log2;
        } else {
#pragma unroll
            for (int e = 0; e < VEC; ++e) qf[g][e] = 0.f;
        }
    }
    float m[GP], l[GP], acc[GP][VEC];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[g][e] = 0.f;
    }

    for (int t = t0 + warp; t < t1; t += NW) {
        const int32_t phys = a.block_tables[(int64_t)b * a.MB + t / a.bs];
        if (phys < 0 || (int64_t)phys >= a.N) {
            if (lane == 0) raise_flag(a.err, PA_DEV_BAD_BLOCK);
            continue;
        }
        const int slot = t % a.bs;
        const int64_t row = (int64_t)phys * a.block_stride + ((int64_t)slot * a.Hkv + h) * D + lane * VEC;
        float kf[VEC], vf[VEC];
        load_kv_row<D, KV>(a.k_cache, row, kf);
        load_kv_row<D, KV>(a.v_cache, row, vf);
        float ks = 1.f, vs = 1.f;
        if constexpr (KV == kKvInt8) {
            const int64_t srow = ((int64_t)phys * a.bs + slot) * a.Hkv + h;
            ks = __ldg(a.k_scale + srow);
            vs = __ldg(a.v_scale + srow);
        }
#pragma unroll
        for (int g = 0; g < GP; ++g) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) s = fmaf(qf[g][e], kf[e], s);
            s = warp_sum(s) * ks;
            const float mn = fmaxf(m[g], s);
            const float alpha = exp2f(m[g] - mn);
            const float p = exp2f(s - mn);
            l[g] = l[g] * alpha + p;
            const float pv = p * vs;
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[g][e] = fmaf(pv, vf[e], acc[g][e] * alpha);
            m[g] = mn;
        }
    }

    __shared__ float sm_m[NW][GP], sm_l[NW][GP];
    __shared__ float sm_acc[NW][GP][D];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
        if (lane == 0) {
            sm_m[warp][g] = m[g];
            sm_l[warp][g] = l[g];
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) sm_acc[warp][g][lane * VEC + e] = acc[g][e];
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < a.G * D; idx += blockDim.x) {
        const int g = idx / D, e = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, sm_m[w][g]);
        float L = 0.f, A = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float f = exp2f(sm_m[w][g] - M);
                L = fmaf(sm_l[w][g], f, L);
                A = fmaf(sm_acc[w][g][e], f, A);
            }
        }
        const int64_t bh = (int64_t)b * a.Hq + h * a.G + g;
        if (a.num_splits == 1) {
            a.out[bh * D + e] = f32_to_bf16_rn(L > 0.f ? A / L : 0.f);
        } else {
            a.ws_acc[(bh * a.num_splits + c) * D + e] = A;
            if (e == 0) {
                a.ws_ml[(bh * a.num_splits + c) * 2 + 0] = M;
                a.ws_ml[(bh * a.num_splits + c) * 2 + 1] = L;
            }
        }
    }
}

// Log-sum-exp merge of the partitions of one (sequence, query head):
// M = max_s m_s, L = sum_s l_s 2^(m_s - M), out = sum_s acc_s 2^(m_s - M) / L.
// Partitions are visited in index order (deterministic, no atomics).
template <int D>
__global__ void __launch_bounds__(D) merge_kernel(DecodeArgs a) {
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / a.Hq);
    const int e = threadIdx.x;
    int len = a.ctx_lens[b];
    if (len < 0 || (int64_t)len > (int64_t)a.MB * a.bs) len = 0;
    const int ns = len > 0 ? (len + a.chunk - 1) / a.chunk : 1;
    const float *ml = a.ws_ml + bh * a.num_splits * 2;
    const float *acc = a.ws_acc + bh * a.num_splits * D;
    float M = -INFINITY;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, ml[2 * s]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < ns; ++s) {
            const float f = exp2f(ml[2 * s] - M);
            L = fmaf(ml[2 * s + 1], f, L);
            A = fmaf(acc[(int64_t)s * D + e], f, A);
        }
    }
    a.out[bh * D + e] = f32_to_bf16_rn(L > 0.f ? A / L : 0.f);
}

template <int D, int KV>
static void launch_simple_gp(const DecodeArgs &a, dim3 grid, cudaStream_t st) {
    int gp = 1;
    while (gp < a.G) gp <<= 1;
    switch (gp) {
        case 1: decode_simple_kernel<D, 1, KV><<<grid, 128, 0, st>>>(a); break;
        case 2: decode_simple_kernel<D, 2, KV><<<grid, 128, 0, st>>>(a); break;
        case 4: decode_simple_kernel<D, 4, KV><<<grid, 128, 0, st>>>(a); break;
        case 8: decode_simple_kernel<D, 8, KV><<<grid, 128, 0, st>>>(a); break;
        default: decode_simple_kernel<D, 16, KV><<<grid, 128, 0, st>>>(a); break;
    }
}

template <int D>
static void launch_simple_kv(const DecodeArgs &a, int kv, dim3 grid, cudaStream_t st) {
    if (kv == kKvInt8) launch_simple_gp<D, kKvInt8>(a, grid, st);
    else if (kv == kKvFp8) launch_simple_gp<D, kKvFp8>(a, grid, st);
    else launch_simple_gp<D, kKvBf16>(a, grid, st);
}

cudaError_t launch_decode_simple(const DecodeArgs &a, int kv, cudaStream_t st) {
    dim3 grid(a.num_splits, a.Hkv, a.B);
    if (a.d == 128) launch_simple_kv<128>(a, kv, grid, st);
    else launch_simple_kv<64>(a, kv, grid, st);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || a.num_splits == 1) return e;
    return launch_merge(a, st);
}

cudaError_t launch_merge(const DecodeArgs &a, cudaStream_t st) {
    const unsigned rows = (unsigned)((int64_t)a.B * a.Hq);
    if (a.d == 128) merge_kernel<128><<<rows, 128, 0, st>>>(a);
    else merge_kernel<64><<<rows, 64, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, int kv, cudaStream_t st) {
    if (a.plan.kernel == 1) return launch_decode_tc(a, kv, st);   // selection included
    cudaError_t e = launch_decode_simple(a, kv, st);
    if (e == cudaSuccess && a.sel_evict)
        e = launch_select_pooled(a.sel_evict, a.sel_means, a.sel_scores, a.block_tables,
                                 a.ctx_lens, a.err, a.B, a.MB, a.Hkv, a.bs, a.N, st);
    return e;
}

namespace {
inline size_t up256(size_t x) { return (x + 255) / 256 * 256; }
inline int up1024(int x) { return (x + 1023) / 1024 * 1024; }
}  // namespace

// Host launch plan.  The staged tensor-core kernel takes pools with a block
// size that is a multiple of 16, Hkv in {1, 2, 4, 8} and G <= 16 (INT8, FP8: d = 128)
// when at least two pipeline stages fit in shared memory; everything else runs
// the general-shape kernel.
DecodePlan make_decode_plan(int B, int Hq, int Hkv, int d, int bs, int MB, int num_splits,
                            int kv, int sms) {
    const bool onebyte = kv != kKvBf16;  // int8 and fp8 pools: one byte per element
    DecodePlan p;
    memset(&p, 0, sizeof p);
    const int64_t max_ctx = (int64_t)MB * bs;
    const int G = Hq / Hkv;
    bool tc = bs % 16 == 0 && (Hkv == 1 || Hkv == 2 || Hkv == 4 || Hkv == 8) && G <= 16 &&
              (!onebyte || d == 128);
    if (tc) {
        const int box = Hkv * 16 * 128;  // one 128-byte slice of d of 16 tokens, all heads
        const int DC = onebyte ? d / 128 : d / 64;
        const int sub_kv = DC * box;                    // K (or V) bytes of one 16-token sub-tile
        const int sub_sc = kv == kKvInt8 ? 16 * Hkv * 4 : 0;  // its scale rows
        p.wph = 8 / Hkv;
        // sub-tiles per warp per stage: stages of about 64 KB of K + V amortise the
        // per-stage cost of the pipeline
        int tpw = 1;
        while (tpw < 4 && p.wph * tpw * 2 <= 32 && 2 * (p.wph * tpw * 2) * sub_kv <= 64 * 1024)
            tpw *= 2;  // doubling keeps the stage (K + V of n_sub sub-tiles) within 64 KB
        p.tpw = tpw;
        p.n_sub = p.wph * tpw;
        // the INT8 and FP8 consumers take a warp's sub-tiles of a stage as one pair
        // (the doubling above gives one-byte pools exactly two)
        if (onebyte && tpw > 2) tc = false;
        const int kv_bytes = p.n_sub * sub_kv;
        const int sc_bytes = p.n_sub * sub_sc;
        p.v_off = kv_bytes;
        p.ks_off = 2 * kv_bytes;
        p.vs_off = p.ks_off + sc_bytes;
        p.stage_bytes = up1024(p.vs_off + sc_bytes);
        const int avail = 227 * 1024 - 1024;
        int ns = avail / (p.stage_bytes + 48);
        if (ns > 8) ns = 8;
        if (ns < 2) tc = false;
        p.nstage = ns;
        p.smem_bytes = ns * p.stage_bytes + ns * 48 + 1024;
    }
    if (tc) {
        p.kernel = 1;
        p.grid = sms;
        p.units_per_cta = 4;
        int64_t mc = 128;
        size_t n_units;
        if (num_splits > 0 || sms >= 1024) {
            // explicit split: at most num_splits near-equal partitions per sequence,
            // taken by the CTAs from a counter, longest first (also the automatic
            // split on a GPU with more SMs than the balanced plan's ranges)
            if (num_splits > 0) mc = ((max_ctx + num_splits - 1) / num_splits + 15) / 16 * 16;
            if (mc < 16) mc = 16;
            p.S = (int)((max_ctx + mc - 1) / mc);
            n_units = (size_t)B * p.S;
        } else {
            // automatic split: the concatenated contexts are cut into one equal range
            // of at least mc tokens per CTA (cuts snapped to 16-token tiles); a
            // sequence holds at most ceil(len / mc) cuts, so at most that many + 1
            // pieces, and all pieces number at most B + grid
            p.balanced = 1;
            p.S = (int)((max_ctx + mc - 1) / mc) + 1;
            n_units = (size_t)B + (size_t)p.grid;
        }
        p.chunk = (int)mc;
        const size_t slots = (size_t)B * p.S * p.wph * Hq;
        p.off_hdr = 0;
        p.off_ns = 256;
        p.off_units = p.off_ns + up256((size_t)B * 4);
        p.off_cta = p.off_units + up256(n_units * 16);
        p.off_first = p.off_cta + up256((size_t)(p.grid + 1) * 4);
        p.off_starts = p.off_first + up256((size_t)p.grid * 16);
        p.off_ml = p.off_starts + up256(p.balanced ? (size_t)B * 8 : 0);
        p.off_acc = p.off_ml + up256(slots * 2 * 4);
        p.ws_total = p.off_acc + up256(slots * d * 4);
        // sizes the device plan depends on (a plan kept in a workspace is only used by
        // calls of the same signature): FNV-1a over them.  The element type is not
        // among them: bf16, INT8 and FP8 calls of the same sizes share one plan.
        const long long f[11] = {B,      Hq,     Hkv,    d,      bs,           MB,
                                 p.S,    p.chunk, p.grid, p.units_per_cta, p.balanced};
        unsigned long long h = 1469598103934665603ull;
        for (long long v : f) {
            h ^= (unsigned long long)v;
            h *= 1099511628211ull;
        }
        p.sig = h | 1ull;  // never 0 (a zeroed workspace holds no plan)
        return p;
    }
    // general-shape kernel: fixed partitions of `chunk` tokens
    int64_t s = num_splits;
    if (s <= 0) {
        const int64_t units = (int64_t)(B > 0 ? B : 1) * Hkv;
        const int64_t target = 4LL * sms;
        s = units >= target ? 1 : (target + units - 1) / units;
        const int64_t cap = (max_ctx + 255) / 256;
        if (s > cap) s = cap;
    }
    if (s < 1) s = 1;
    if (s > max_ctx) s = max_ctx;
    int64_t ch = (max_ctx + s - 1) / s;
    ch = (ch + 15) / 16 * 16;
    const int64_t se = (max_ctx + ch - 1) / ch;
    p.kernel = 0;
    p.S = (int)se;
    p.chunk = (int)(se == 1 ? max_ctx : ch);
    if (p.S > 1) {
        const size_t rows = (size_t)B * Hq * p.S;
        p.off_acc = 0;
        p.off_ml = up256(rows * d * 4);
        p.ws_total = p.off_ml + up256(rows * 2 * 4);
    }
    return p;
}

}  // namespace pkv
