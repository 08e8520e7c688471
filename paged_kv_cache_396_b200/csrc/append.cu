// append.cu -- KV append (scatter of new tokens into the paged pools), bf16 and
// quantising INT8.
//
// Slot of position p in sequence b: block_tables[b][p / bs] * bs + p % bs
// (ybb.press "LLM 推理 KV Cache 内存管理深度工程实践" §2.1, append_slot).
// INT8 rows follow §6.1 of the same page: s = amax / 127, code = round(x / s).
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
template <int D>
__global__ void append_int8_kernel(const uint16_t *__restrict__ k_new,
                                   const uint16_t *__restrict__ v_new, int8_t *__restrict__ kq,
                                   int8_t *__restrict__ vq, float *__restrict__ k_scale,
                                   float *__restrict__ v_scale, AppendArgs a) {
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
        float s;
        load_row<D>(k_new + src, x);
        quantise_row<PER>(x, q, s);
        store_codes<D>(kq + dst, q);
        if (lane == 0) k_scale[sdst] = s;
        load_row<D>(v_new + src, x);
        quantise_row<PER>(x, q, s);
        store_codes<D>(vq + dst, q);
        if (lane == 0) v_scale[sdst] = s;
        if (leader && a.slot_out) a.slot_out[bi] = (int64_t)phys * a.bs + off;
    }
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
                               int8_t *vq, float *k_scale, float *v_scale, const AppendArgs &a,
                               int num_sms, cudaStream_t stream) {
    const int64_t rows = (int64_t)a.B * a.n_new * a.Hkv;
    const int threads = 256;
    int64_t blocks = (rows * 32 + threads - 1) / threads;
    blocks = blocks < (int64_t)num_sms * 16 ? blocks : (int64_t)num_sms * 16;
    if (a.d == 128)
        append_int8_kernel<128><<<(unsigned)blocks, threads, 0, stream>>>(k_new, v_new, kq, vq,
                                                                          k_scale, v_scale, a);
    else
        append_int8_kernel<64><<<(unsigned)blocks, threads, 0, stream>>>(k_new, v_new, kq, vq,
                                                                         k_scale, v_scale, a);
    return cudaGetLastError();
}

}  // namespace pkv
