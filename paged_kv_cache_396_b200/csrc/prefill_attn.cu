// prefill_attn.cu -- multi-query paged attention for a chunked prefill.
//
// t6page.pages.dev "KV cache", "Chunked prefill：让 prefill 不阻塞 decode": a long
// prompt is prefilled in chunks (512 tokens) batched with the running decodes;
// each chunk's queries attend, through the block table ("PagedAttention 的算子"),
// every cached token of their sequence up to their own position.  The chunk's
// K/V rows are appended first (pa_append_kv with n_new = chunk length), so the
// q_len query tokens of a sequence are its last q_len cached tokens.
//
// The work is a dense contraction (q_len x G query rows against the whole
// context), so it runs on tensor cores.  One CTA = one (sequence, kv head,
// tile of 64 query rows): rows are (query token, head of the GQA group) pairs,
// G heads of one token adjacent, so every K/V tile loaded serves all G heads.
// Four warps own 16 rows each.  K/V tiles of 64 tokens are gathered through
// the block table with cp.async into a two-stage, XOR-swizzled shared buffer;
// S = Q K^T and O += P V use mma.m16n8k16 (bf16 in, fp32 accumulate) with the
// softmax online in the exp2 domain; P stays in registers as the A operand of
// the second product, split into two bf16 parts (hi + lo) so that the weights
// keep ~16 bits.  Query tiles are issued longest-context first.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "prefill_attn.h"
#include "ptx.cuh"

namespace pkv {

namespace {

constexpr int kRows = 64;       // query rows per CTA (4 warps x 16)
constexpr int kThreads = 128;
constexpr int kKT = 64;         // tokens per K/V tile
constexpr unsigned kFullMask = 0xffffffffu;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    // src-size 0 fills the 16 bytes with zeros and reads nothing
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Row of 16-byte chunks c of token row r in a swizzled tile (ROWB bytes per row).
template <int ROWB>
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return (uint32_t)(r * ROWB + ((c ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kThreads, 3) prefill_attn_kernel(const PrefillAttnArgs a) {
    constexpr int ROWB = D * 2;          // bytes per token row of one head
    constexpr int CH = ROWB / 16;        // 16-byte chunks per row
    constexpr int TILEB = kKT * ROWB;    // one K (or V) tile
    constexpr int NK = D / 16;           // k-steps of Q K^T
    constexpr int NO = D / 8;            // n-tiles of O
    extern __shared__ __align__(128) uint8_t smem[];

    const int b = blockIdx.z, h = blockIdx.y;
    const int G = a.G, QT = kRows / G;   // query tokens per CTA
    const int q0 = a.cu_q[b], ql = a.cu_q[b + 1] - q0;
    const int n_qt = (ql + QT - 1) / QT;
    const int qt = n_qt - 1 - (int)blockIdx.x;   // longest context first
    if (qt < 0) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tig = lane & 3;
    const int len = a.ctx_lens[b];
    const bool bad = len < 0 || (int64_t)len > (int64_t)a.MB * a.bs || ql > len;
    // CTA rows r = i*G + gh: query token qt*QT + i, head h*G + gh
    const int tok_base = qt * QT;
    const int pos0 = len - ql;           // position of query token 0
    // this thread's two rows (g and g + 8 of its warp's 16)
    const int rA = warp * 16 + g, rB = rA + 8;
    const int iA = tok_base + rA / G, iB = tok_base + rB / G;
    const bool vA = iA < ql && !bad, vB = iB < ql && !bad;
    const int pA = pos0 + iA, pB = pos0 + iB;   // causal limits (inclusive)
    if (bad) {
        // invalid sequence: zero output rows, flag once
        if (blockIdx.x == 0 && h == 0 && tid == 0) raise_flag(a.err, PA_DEV_BAD_LEN);
        for (int r = warp; r < kRows; r += 4) {
            const int i = tok_base + r / G;
            if (i >= ql) continue;
            uint16_t *o = a.out + ((int64_t)(q0 + i) * a.Hq + h * G + r % G) * D;
            for (int e = lane; e < D; e += 32) o[e] = 0;
        }
        return;
    }
    const int last_tok = min(ql - 1, tok_base + QT - 1);
    const int p_max = pos0 + last_tok;                  // highest position in this CTA
    const int n_kt = p_max / kKT + 1;                   // K/V tiles to visit

    // ---- Q fragments (A operand), straight from global: rows rA and rB
    uint32_t qa[NK][4];
    {
        const uint32_t *qrA = reinterpret_cast<const uint32_t *>(
            a.q + ((int64_t)(q0 + min(iA, ql - 1)) * a.Hq + h * G + rA % G) * D);
        const uint32_t *qrB = reinterpret_cast<const uint32_t *>(
            a.q + ((int64_t)(q0 + min(iB, ql - 1)) * a.Hq + h * G + rB % G) * D);
#pragma unroll
        for (int kk = 0; kk < NK; ++kk) {
            qa[kk][0] = qrA[kk * 8 + tig];
            qa[kk][1] = qrB[kk * 8 + tig];
            qa[kk][2] = qrA[kk * 8 + 4 + tig];
            qa[kk][3] = qrB[kk * 8 + 4 + tig];
        }
    }

    const uint32_t sbase = ptx::smem_u32(smem);
    const int32_t *btr = a.block_tables + (int64_t)b * a.MB;
    // stage s: K tile at s*2*TILEB, V tile at s*2*TILEB + TILEB
    auto load_tile = [&](int kt, int s) {
        const uint32_t kdst = sbase + (uint32_t)(s * 2 * TILEB);
        const uint32_t vdst = kdst + TILEB;
#pragma unroll
        for (int k = 0; k < kKT * CH / kThreads; ++k) {
            const int idx = tid + k * kThreads;
            const int r = idx / CH, c = idx % CH;
            const int t = kt * kKT + r;
            bool ok = t < len;
            const int64_t blk = ok ? btr[t / a.bs] : 0;
            if (ok && (blk < 0 || blk >= a.N)) {
                raise_flag(a.err, PA_DEV_BAD_BLOCK);
                ok = false;
            }
            const int64_t off =
                ok ? blk * a.block_stride + ((int64_t)(t % a.bs) * a.Hkv + h) * D + c * 8 : 0;
            cp_async16(kdst + swz<ROWB>(r, c), a.k_cache + off, ok);
            cp_async16(vdst + swz<ROWB>(r, c), a.v_cache + off, ok);
        }
        cp_async_commit();
    };

    float o[NO][4];
#pragma unroll
    for (int j = 0; j < NO; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    const float sl = a.scale_log2;

    load_tile(0, 0);
    for (int kt = 0; kt < n_kt; ++kt) {
        const int s = kt & 1;
        if (kt + 1 < n_kt) {
            load_tile(kt + 1, s ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const uint32_t kt_s = sbase + (uint32_t)(s * 2 * TILEB);
        const uint32_t vt_s = kt_s + TILEB;

        // ---- S = Q K^T over 64 tokens: 8 n-tiles of 8 tokens
        float sc[kKT / 8][4];
#pragma unroll
        for (int j = 0; j < kKT / 8; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
        for (int j = 0; j < kKT / 8; ++j) {
#pragma unroll
            for (int kk = 0; kk < NK; kk += 2) {
                // 4 matrices: (tokens 8j.., dims 16kk.. lo/hi), (.., 16(kk+1).. lo/hi)
                const int mi = lane >> 3, rr = lane & 7;
                uint32_t bfr[4];
                ptx::ldmatrix_x4(bfr, kt_s + swz<ROWB>(8 * j + rr, 2 * kk + mi));
                ptx::mma_bf16(sc[j], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], bfr[0], bfr[1]);
                ptx::mma_bf16(sc[j], qa[kk + 1][0], qa[kk + 1][1], qa[kk + 1][2], qa[kk + 1][3],
                              bfr[2], bfr[3]);
            }
        }
        // ---- causal mask (only where the tile reaches past the row's position)
        const int t0 = kt * kKT;
        float xA = -INFINITY, xB = -INFINITY;
#pragma unroll
        for (int j = 0; j < kKT / 8; ++j) {
            const int tc = t0 + 8 * j + 2 * tig;
            sc[j][0] = (vA && tc <= pA) ? sc[j][0] * sl : -INFINITY;
            sc[j][1] = (vA && tc + 1 <= pA) ? sc[j][1] * sl : -INFINITY;
            sc[j][2] = (vB && tc <= pB) ? sc[j][2] * sl : -INFINITY;
            sc[j][3] = (vB && tc + 1 <= pB) ? sc[j][3] * sl : -INFINITY;
            xA = fmaxf(xA, fmaxf(sc[j][0], sc[j][1]));
            xB = fmaxf(xB, fmaxf(sc[j][2], sc[j][3]));
        }
        xA = fmaxf(xA, __shfl_xor_sync(kFullMask, xA, 1));
        xA = fmaxf(xA, __shfl_xor_sync(kFullMask, xA, 2));
        xB = fmaxf(xB, __shfl_xor_sync(kFullMask, xB, 1));
        xB = fmaxf(xB, __shfl_xor_sync(kFullMask, xB, 2));
        const float nA = fmaxf(mA, xA), nB = fmaxf(mB, xB);
        const float uA = nA == -INFINITY ? 0.f : nA, uB = nB == -INFINITY ? 0.f : nB;
        const float alA = exp2f(mA - uA), alB = exp2f(mB - uB);
        mA = nA;
        mB = nB;
        float sA = 0.f, sB = 0.f;
#pragma unroll
        for (int j = 0; j < kKT / 8; ++j) {
            sc[j][0] = exp2f(sc[j][0] - uA);
            sc[j][1] = exp2f(sc[j][1] - uA);
            sc[j][2] = exp2f(sc[j][2] - uB);
            sc[j][3] = exp2f(sc[j][3] - uB);
            sA += sc[j][0] + sc[j][1];
            sB += sc[j][2] + sc[j][3];
        }
        lA = lA * alA + sA;
        lB = lB * alB + sB;
#pragma unroll
        for (int j = 0; j < NO; ++j) {
            o[j][0] *= alA;
            o[j][1] *= alA;
            o[j][2] *= alB;
            o[j][3] *= alB;
        }
        // ---- O += P V: 4 k-steps of 16 tokens, NO n-tiles of 8 dims.  P = hi + lo in
        // bf16 (p - hi is exact in fp32): a single bf16 weight can be off by 2^-9 of
        // itself, too coarse when a few tokens hold most of the weight.
#pragma unroll
        for (int kk = 0; kk < kKT / 16; ++kk) {
            const float(&s0)[4] = sc[2 * kk];
            const float(&s1)[4] = sc[2 * kk + 1];
            const uint32_t a0 = ptx::pack_bf16(s0[0], s0[1]), a1 = ptx::pack_bf16(s0[2], s0[3]);
            const uint32_t a2 = ptx::pack_bf16(s1[0], s1[1]), a3 = ptx::pack_bf16(s1[2], s1[3]);
            const uint32_t b0 = ptx::pack_bf16(s0[0] - bf16_lo(a0), s0[1] - bf16_hi(a0));
            const uint32_t b1 = ptx::pack_bf16(s0[2] - bf16_lo(a1), s0[3] - bf16_hi(a1));
            const uint32_t b2 = ptx::pack_bf16(s1[0] - bf16_lo(a2), s1[1] - bf16_hi(a2));
            const uint32_t b3 = ptx::pack_bf16(s1[2] - bf16_lo(a3), s1[3] - bf16_hi(a3));
#pragma unroll
            for (int j = 0; j < NO; j += 2) {
                // 4 matrices: (tokens 16kk.. lo/hi) x (dims 8j.., 8(j+1)..), transposed
                const int mi = lane >> 3, rr = lane & 7;
                const int tr = 16 * kk + 8 * (mi & 1) + rr;
                uint32_t bfr[4];
                ptx::ldmatrix_x4_trans(bfr, vt_s + swz<ROWB>(tr, j + (mi >> 1)));
                ptx::mma_bf16(o[j], a0, a1, a2, a3, bfr[0], bfr[1]);
                ptx::mma_bf16(o[j + 1], a0, a1, a2, a3, bfr[2], bfr[3]);
                ptx::mma_bf16(o[j], b0, b1, b2, b3, bfr[0], bfr[1]);
                ptx::mma_bf16(o[j + 1], b0, b1, b2, b3, bfr[2], bfr[3]);
            }
        }
        __syncthreads();  // this stage is refilled two tiles later
    }

    // ---- normalise and store
    lA += __shfl_xor_sync(kFullMask, lA, 1);
    lA += __shfl_xor_sync(kFullMask, lA, 2);
    lB += __shfl_xor_sync(kFullMask, lB, 1);
    lB += __shfl_xor_sync(kFullMask, lB, 2);
    const float invA = lA > 0.f ? 1.f / lA : 0.f, invB = lB > 0.f ? 1.f / lB : 0.f;
    if (vA) {
        uint32_t *orow = reinterpret_cast<uint32_t *>(
            a.out + ((int64_t)(q0 + iA) * a.Hq + h * G + rA % G) * D);
#pragma unroll
        for (int j = 0; j < NO; ++j)
            orow[4 * j + tig] = (uint32_t)f32_to_bf16_rn(o[j][0] * invA) |
                                ((uint32_t)f32_to_bf16_rn(o[j][1] * invA) << 16);
    }
    if (vB) {
        uint32_t *orow = reinterpret_cast<uint32_t *>(
            a.out + ((int64_t)(q0 + iB) * a.Hq + h * G + rB % G) * D);
#pragma unroll
        for (int j = 0; j < NO; ++j)
            orow[4 * j + tig] = (uint32_t)f32_to_bf16_rn(o[j][2] * invB) |
                                ((uint32_t)f32_to_bf16_rn(o[j][3] * invB) << 16);
    }
}

template <int D>
cudaError_t launch_typed(const PrefillAttnArgs &a, int max_q_len, cudaStream_t st) {
    constexpr int smem = 2 * 2 * kKT * D * 2;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(prefill_attn_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const int QT = kRows / a.G;
    dim3 grid((unsigned)((max_q_len + QT - 1) / QT), (unsigned)a.Hkv, (unsigned)a.B);
    prefill_attn_kernel<D><<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_attn(const PrefillAttnArgs &a, int max_q_len, cudaStream_t st) {
    if (a.d == 128) return launch_typed<128>(a, max_q_len, st);
    if (a.d == 64) return launch_typed<64>(a, max_q_len, st);
    return cudaErrorInvalidValue;
}

}  // namespace pkv
