// append.cu -- KV append (scatter of new tokens into the paged pools), bf16 and
// quantising INT8.
//
// Slot of position p in sequence b: block_tables[b][p / bs] * bs + p % bs
// (ybb.press "LLM 推理 KV Cache 内存管理深度工程实践" §2.1, append_slot).
// INT8 rows follow §6.1 of the same page: s = amax / 127, code = round(x / s).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace pkv {

// One thread per 16-byte chunk of a (sequence, token, kv head) row: the source
// [B][n_new][Hkv][d] is read fully coalesced; each destination row is d*2
// contiguous bytes in the pool.
__global__ void append_bf16_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                                   uint16_t *__restrict__ k_cache, uint16_t *__restrict__ v_cache,
                                   AppendArgs a) {
    const int vec_per_row = a.d / 8;
    const int64_t total = (int64_t)a.B * a.n_new * a.Hkv * vec_per_row;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int c = (int)(idx % vec_per_row);
        const int64_t row = idx / vec_per_row;
        const int h = (int)(row % a.Hkv);
        const int64_t bi = row / a.Hkv;  // b * n_new + i
        const int i = (int)(bi % a.n_new);
        const int b = (int)(bi / a.n_new);
        const bool leader = (h == 0 && c == 0);
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
        const int64_t dst = (int64_t)phys * a.block_stride + (off * a.Hkv + h) * a.d + c * 8;
        *reinterpret_cast<uint4 *>(k_cache + dst) = __ldg(k_new + idx);
        *reinterpret_cast<uint4 *>(v_cache + dst) = __ldg(v_new + idx);
        if (leader && a.slot_out) a.slot_out[bi] = (int64_t)phys * a.bs + off;
    }
}

// Quantise one row of D bf16 values spread over a warp (PER = D/32 per lane).
template <int PER>
__device__ __forceinline__ void quantise_row(const float (&x)[PER], int8_t (&q)[PER], float &s) {
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) amax = fmaxf(amax, fabsf(x[e]));
    amax = warp_max(amax);
    s = __fdiv_rn(amax, 127.0f);  // one correctly rounded fp32 division
#pragma unroll
    for (int e = 0; e < PER; ++e)
        q[e] = (s == 0.f) ? (int8_t)0 : (int8_t)__float2int_rn(__fdiv_rn(x[e], s));
}

template <int D>
__device__ __forceinline__ void load_row(const uint16_t *p, float (&x)[D / 32]) {
    constexpr int PER = D / 32;
    if constexpr (PER == 4) {
        uint2 w = __ldg(reinterpret_cast<const uint2 *>(p));
        x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    } else {
        static_assert(PER == 2, "d must be 64 or 128");
        uint32_t w = __ldg(reinterpret_cast<const unsigned int *>(p));
        x[0] = bf16_lo(w); x[1] = bf16_hi(w);
    }
}

template <int D>
__device__ __forceinline__ void store_codes(int8_t *p, const int8_t (&q)[D / 32]) {
    constexpr int PER = D / 32;
    if constexpr (PER == 4) {
        uint32_t w = (uint32_t)(uint8_t)q[0] | ((uint32_t)(uint8_t)q[1] << 8) |
                     ((uint32_t)(uint8_t)q[2] << 16) | ((uint32_t)(uint8_t)q[3] << 24);
        *reinterpret_cast<uint32_t *>(p) = w;
    } else {
        uint16_t w = (uint16_t)((uint32_t)(uint8_t)q[0] | ((uint32_t)(uint8_t)q[1] << 8));
        *reinterpret_cast<uint16_t *>(p) = w;
    }
}

// One warp per (sequence, token, kv head) row: amax by warp reduction, then
// the per-element code; lane 0 stores the row's scale.
// score_pool (nullable): also store ||V||_2 / ||K||_2 of the dequantised row
// (PagedEviction importance, see score_pool.cu) at the row's slot.
template <int D>
__global__ void append_int8_kernel(const uint16_t *__restrict__ k_new,
                                   const uint16_t *__restrict__ v_new, int8_t *__restrict__ kq,
                                   int8_t *__restrict__ vq, float *__restrict__ k_scale,
                                   float *__restrict__ v_scale, float *__restrict__ score_pool,
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
        const int64_t sdst = ((int64_t)phys * a.bs + off) * a.Hkv + h;
        float x[PER];
        int8_t q[PER];
        float s, kk = 0.f, vv = 0.f;
        load_row<D>(k_new + src, x);
        quantise_row<PER>(x, q, s);
        store_codes<D>(kq + dst, q);
        if (lane == 0) k_scale[sdst] = s;
        if (score_pool) {
#pragma unroll
            for (int e = 0; e < PER; ++e) {
                const float y = s * (float)q[e];
                kk = fmaf(y, y, kk);
            }
        }
        load_row<D>(v_new + src, x);
        quantise_row<PER>(x, q, s);
        store_codes<D>(vq + dst, q);
        if (lane == 0) v_scale[sdst] = s;
        if (score_pool) {
#pragma unroll
            for (int e = 0; e < PER; ++e) {
                const float y = s * (float)q[e];
                vv = fmaf(y, y, vv);
            }
            kk = warp_sum(kk);
            vv = warp_sum(vv);
            if (lane == 0)
                score_pool[sdst] = kk == 0.f ? (vv > 0.f ? INFINITY : 0.f) : sqrtf(vv) / sqrtf(kk);
        }
        if (leader && a.slot_out) a.slot_out[bi] = (int64_t)phys * a.bs + off;
    }
}

// FP8 append ([VKV] §6.1 FP8 branch: a cast of the KV to float8_e4m3fn).  One
// thread per 8 elements of a (sequence, token, kv head) row: 16 bytes of bf16
// in, 8 bytes of e4m3 out, each pair converted round-to-nearest-even with
// saturation at +-448 (cvt.rn.satfinite.e4m3x2.f32).
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__global__ void append_fp8_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                                  uint8_t *__restrict__ k8, uint8_t *__restrict__ v8, AppendArgs a) {
    const int vec_per_row = a.d / 8;
    const int64_t total = (int64_t)a.B * a.n_new * a.Hkv * vec_per_row;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int c = (int)(idx % vec_per_row);
        const int64_t row = idx / vec_per_row;
        const int h = (int)(row % a.Hkv);
        const int64_t bi = row / a.Hkv;
        const int i = (int)(bi % a.n_new);
        const int b = (int)(bi / a.n_new);
        const bool leader = (h == 0 && c == 0);
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
        const int64_t dst = (int64_t)phys * a.block_stride + (off * a.Hkv + h) * a.d + c * 8;
        const uint4 kw = __ldg(k_new + idx), vw = __ldg(v_new + idx);
        const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w}, vv[4] = {vw.x, vw.y, vw.z, vw.w};
        uint32_t ko[2], vo[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            ko[q] = f32x2_to_e4m3x2(bf16_lo(kk[2 * q]), bf16_hi(kk[2 * q])) |
                    (f32x2_to_e4m3x2(bf16_lo(kk[2 * q + 1]), bf16_hi(kk[2 * q + 1])) << 16);
            vo[q] = f32x2_to_e4m3x2(bf16_lo(vv[2 * q]), bf16_hi(vv[2 * q])) |
                    (f32x2_to_e4m3x2(bf16_lo(vv[2 * q + 1]), bf16_hi(vv[2 * q + 1])) << 16);
        }
        *reinterpret_cast<uint2 *>(k8 + dst) = make_uint2(ko[0], ko[1]);
        *reinterpret_cast<uint2 *>(v8 + dst) = make_uint2(vo[0], vo[1]);
        if (leader && a.slot_out) a.slot_out[bi] = (int64_t)phys * a.bs + off;
    }
}

cudaError_t launch_append_fp8(const uint16_t *k_new, const uint16_t *v_new, uint8_t *k8,
                              uint8_t *v8, const AppendArgs &a, int num_sms, cudaStream_t stream) {
    const int64_t total = (int64_t)a.B * a.n_new * a.Hkv * (a.d / 8);
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    blocks = blocks < (int64_t)num_sms * 16 ? blocks : (int64_t)num_sms * 16;
    append_fp8_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
        reinterpret_cast<const uint4 *>(k_new), reinterpret_cast<const uint4 *>(v_new), k8, v8, a);
    return cudaGetLastError();
}

cudaError_t launch_append_bf16(const uint16_t *k_new, const uint16_t *v_new, uint16_t *k_cache,
                               uint16_t *v_cache, const AppendArgs &a, int num_sms,
                               cudaStream_t stream) {
    const int64_t total = (int64_t)a.B * a.n_new * a.Hkv * (a.d / 8);
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    blocks = blocks < (int64_t)num_sms * 16 ? blocks : (int64_t)num_sms * 16;
    append_bf16_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
        reinterpret_cast<const uint4 *>(k_new), reinterpret_cast<const uint4 *>(v_new), k_cache,
        v_cache, a);
    return cudaGetLastError();
}

cudaError_t launch_append_int8(const uint16_t *k_new, const uint16_t *v_new, int8_t *kq,
                               int8_t *vq, float *k_scale, float *v_scale, float *score_pool,
                               const AppendArgs &a, int num_sms, cudaStream_t stream) {
    const int64_t rows = (int64_t)a.B * a.n_new * a.Hkv;
    const int threads = 256;
    int64_t blocks = (rows * 32 + threads - 1) / threads;
    blocks = blocks < (int64_t)num_sms * 16 ? blocks : (int64_t)num_sms * 16;
    if (a.d == 128)
        append_int8_kernel<128><<<(unsigned)blocks, threads, 0, stream>>>(
            k_new, v_new, kq, vq, k_scale, v_scale, score_pool, a);
    else
        append_int8_kernel<64><<<(unsigned)blocks, threads, 0, stream>>>(
            k_new, v_new, kq, vq, k_scale, v_scale, score_pool, a);
    return cudaGetLastError();
}

}  // namespace pkv
