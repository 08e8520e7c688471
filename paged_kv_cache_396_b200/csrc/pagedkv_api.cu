// pagedkv_api.cu -- the extern "C" entry points declared in include/pagedkv.h:
// argument validation, launch-shape decisions and kernel launches.  Nothing
// here allocates device memory or keeps state between calls beyond a per-device
// cache of the SM count.
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "kernels.h"
#include "prefill.h"
#include "prefill_attn.h"
#include "selftest.h"
#include "pagedkv.h"

namespace {

struct DevCache {
    std::atomic<int> sms{0};
    std::atomic<int> major{0};
};
DevCache g_dev[64];

// Current device's SM count, or a negative PA_ERR_* when it is not an sm_100 GPU.
int device_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    if (dev < 0 || dev >= 64) return PA_ERR_DEVICE;
    int sms = g_dev[dev].sms.load(std::memory_order_relaxed);
    if (sms == 0) {
        int major = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return PA_ERR_CUDA;
        g_dev[dev].major.store(major);
        g_dev[dev].sms.store(sms);
    }
    if (g_dev[dev].major.load() != 10) return PA_ERR_DEVICE;
    return sms;
}

inline bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int B, int Hkv, int d, int bs, int MB, int64_t N, int64_t block_stride) {
    if (B < 0 || Hkv < 1 || bs < 1 || MB < 1 || N < 1) return PA_ERR_SHAPE;
    if (B > 65535 || Hkv > 65535) return PA_ERR_SHAPE;  // grid y/z limits
    if (d != 64 && d != 128) return PA_ERR_SHAPE;
    if ((int64_t)MB * bs > INT32_MAX) return PA_ERR_SHAPE;
    if (block_stride < (int64_t)bs * Hkv * d) return PA_ERR_SHAPE;
    if (N > INT32_MAX) return PA_ERR_SHAPE;
    return PA_OK;
}

int finish(cudaError_t e) { return e == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

// Shared body of pa_decode / pa_decode_int8.
int decode_entry(uint16_t *out, const uint16_t *q, const void *kc, const void *vc, const float *ks,
                 const float *vs, int kv, int64_t block_stride, const int32_t *bt, int MB,
                 const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs, int64_t N,
                 float scale, int num_splits, void *ws, size_t ws_bytes, int32_t *err,
                 void *stream, int reuse_plan = 0, int32_t *sel_evict = nullptr,
                 float *sel_means = nullptr, const float *sel_scores = nullptr) {
    if (B == 0) return PA_OK;  // empty batch: nothing to read or write
    if (!out || !q || !kc || !vc || !bt || !ctx_lens || !err) return PA_ERR_NULL;
    if (kv == pkv::kKvInt8 && (!ks || !vs)) return PA_ERR_NULL;
    int rc = check_common(B, Hkv, d, bs, MB, N, block_stride);
    if (rc) return rc;
    if (Hq < Hkv || Hq % Hkv != 0 || Hq / Hkv > 16) return PA_ERR_SHAPE;
    if (!(scale == scale)) return PA_ERR_SHAPE;
    const int elt = kv == pkv::kKvBf16 ? 2 : 1;
    if (!al16(out) || !al16(q) || !al16(kc) || !al16(vc) || (block_stride * elt) % 16 != 0)
        return PA_ERR_ALIGN;
    // the staged kernel bulk-copies each tile's scales (cp.async.bulk: 16-byte source)
    if (kv == pkv::kKvInt8 && (!al16(ks) || !al16(vs))) return PA_ERR_ALIGN;
    const int sms = device_sms();
    if (sms < 0) return sms;
    const pkv::DecodePlan plan = pkv::make_decode_plan(B, Hq, Hkv, d, bs, MB, num_splits, kv, sms);
    if (plan.ws_total > 0) {
        if (!ws) return PA_ERR_WORKSPACE;
        if (ws_bytes < plan.ws_total) return PA_ERR_WORKSPACE;
        if (!al16(ws)) return PA_ERR_ALIGN;
    }
    pkv::DecodeArgs a;
    memset(&a, 0, sizeof a);
    a.out = out;
    a.q = q;
    a.k_cache = kc;
    a.v_cache = vc;
    a.k_scale = ks;
    a.v_scale = vs;
    a.block_tables = bt;
    a.ctx_lens = ctx_lens;
    a.err = err;
    a.ws = ws;
    a.plan = plan;
    a.ws_acc = plan.ws_total ? reinterpret_cast<float *>(static_cast<char *>(ws) + plan.off_acc)
                             : nullptr;
    a.ws_ml = plan.ws_total ? reinterpret_cast<float *>(static_cast<char *>(ws) + plan.off_ml)
                            : nullptr;
    a.block_stride = block_stride;
    a.N = N;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.G = Hq / Hkv;
    a.d = d;
    a.bs = bs;
    a.MB = MB;
    a.num_splits = plan.S;
    a.chunk = plan.chunk;
    a.reuse_plan = reuse_plan;
    a.sel_evict = sel_evict;
    a.sel_means = sel_means;
    a.sel_scores = sel_scores;
    return finish(pkv::launch_decode(a, kv, static_cast<cudaStream_t>(stream)));
}

}  // namespace

// Scratch for pa_decode_static_scratch: a fixed array inside the library, one
// copy on every device that loads it, held until the process exits.  In host code
// the name g_static_scratch is a host-side stand-in, not a device address; the
// address comes from static_scratch_address().
static __device__ __align__(256) unsigned char g_static_scratch[PA_STATIC_SCRATCH_BYTES];

namespace {

// Device address of g_static_scratch on the current device, or nullptr on failure.
// Looked up on every call, with the calling device current: a host-side lookup
// that allocates nothing, and stays right when the context is reset and the
// library's device code is loaded again at another address.
void *static_scratch_address() {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
    return p;
}

}  // namespace

extern "C" {

const char *pa_status_string(int code) {
    switch (code) {
        case PA_OK: return "ok";
        case PA_ERR_NULL: return "a required pointer is NULL";
        case PA_ERR_SHAPE: return "unsupported or inconsistent sizes";
        case PA_ERR_ALIGN: return "pointer or stride not 16-byte aligned";
        case PA_ERR_WORKSPACE: return "workspace missing or too small";
        case PA_ERR_CUDA: return "CUDA runtime call or kernel launch failed";
        case PA_ERR_DEVICE: return "current device is not an sm_100 GPU";
        default: return "unknown status";
    }
}

const char *pa_version(void) { return "pagedkv 0.1 sm_100a"; }

int pa_append_kv(const uint16_t *k_new, const uint16_t *v_new, uint16_t *k_cache,
                 uint16_t *v_cache, int64_t block_stride, const int32_t *block_tables,
                 int max_blocks_per_seq, const int32_t *positions, int B, int n_new, int Hkv,
                 int d, int bs, int64_t num_blocks, int64_t *slot_out, int32_t *err_flag,
                 void *stream) {
    if (B == 0 || n_new == 0) return PA_OK;
    if (!k_new || !v_new || !k_cache || !v_cache || !block_tables || !positions || !err_flag)
        return PA_ERR_NULL;
    int rc = check_common(B, Hkv, d, bs, max_blocks_per_seq, num_blocks, block_stride);
    if (rc) return rc;
    if (n_new < 0) return PA_ERR_SHAPE;
    if (!al16(k_new) || !al16(v_new) || !al16(k_cache) || !al16(v_cache) ||
        (block_stride * 2) % 16 != 0)
        return PA_ERR_ALIGN;
    const int sms = device_sms();
    if (sms < 0) return sms;
    pkv::AppendArgs a{block_tables, positions, slot_out, err_flag, block_stride, num_blocks,
                      B, n_new, Hkv, d, bs, max_blocks_per_seq};
    return finish(pkv::launch_append_bf16(k_new, v_new, k_cache, v_cache, a, sms,
                                          static_cast<cudaStream_t>(stream)));
}

int pa_append_kv_int8(const uint16_t *k_new, const uint16_t *v_new, int8_t *kq_cache,
                      int8_t *vq_cache, float *k_scale, float *v_scale, int64_t block_stride,
                      const int32_t *block_tables, int max_blocks_per_seq,
                      const int32_t *positions, int B, int n_new, int Hkv, int d, int bs,
                      int64_t num_blocks, int64_t *slot_out, int32_t *err_flag, void *stream) {
    if (B == 0 || n_new == 0) return PA_OK;
    if (!k_new || !v_new || !kq_cache || !vq_cache || !k_scale || !v_scale || !block_tables ||
        !positions || !err_flag)
        return PA_ERR_NULL;
    int rc = check_common(B, Hkv, d, bs, max_blocks_per_seq, num_blocks, block_stride);
    if (rc) return rc;
    if (n_new < 0) return PA_ERR_SHAPE;
    if (!al16(k_new) || !al16(v_new) || !al16(kq_cache) || !al16(vq_cache) || !al16(k_scale) ||
        !al16(v_scale) || block_stride % 16 != 0)
        return PA_ERR_ALIGN;
    const int sms = device_sms();
    if (sms < 0) return sms;
    pkv::AppendArgs a{block_tables, positions, slot_out, err_flag, block_stride, num_blocks,
                      B, n_new, Hkv, d, bs, max_blocks_per_seq};
    return finish(pkv::launch_append_int8(k_new, v_new, kq_cache, vq_cache, k_scale, v_scale,
                                          nullptr, a, sms, static_cast<cudaStream_t>(stream)));
}

int pa_append_kv_scored(const uint16_t *k_new, const uint16_t *v_new, uint16_t *k_cache,
                        uint16_t *v_cache, int64_t block_stride, float *score_pool,
                        const int32_t *block_tables, int max_blocks_per_seq,
                        const int32_t *positions, int B, int n_new, int Hkv, int d, int bs,
                        int64_t num_blocks, int64_t *slot_out, int32_t *err_flag, void *stream) {
    if (B == 0 || n_new == 0) return PA_OK;
    if (!k_new || !v_new || !k_cache || !v_cache || !score_pool || !block_tables || !positions ||
        !err_flag)
        return PA_ERR_NULL;
    int rc = check_common(B, Hkv, d, bs, max_blocks_per_seq, num_blocks, block_stride);
    if (rc) return rc;
    if (n_new < 0) return PA_ERR_SHAPE;
    if (!al16(k_new) || !al16(v_new) || !al16(k_cache) || !al16(v_cache) ||
        (block_stride * 2) % 16 != 0)
        return PA_ERR_ALIGN;
    const int sms = device_sms();
    if (sms < 0) return sms;
    pkv::AppendArgs a{block_tables, positions, slot_out, err_flag, block_stride, num_blocks,
                      B, n_new, Hkv, d, bs, max_blocks_per_seq};
    return finish(pkv::launch_append_scored(k_new, v_new, k_cache, v_cache, score_pool, a, sms,
                                            static_cast<cudaStream_t>(stream)));
}

int pa_append_kv_int8_scored(const uint16_t *k_new, const uint16_t *v_new, int8_t *kq_cache,
                             int8_t *vq_cache, float *k_scale, float *v_scale, float *score_pool,
                             int64_t block_stride, const int32_t *block_tables,
                             int max_blocks_per_seq, const int32_t *positions, int B, int n_new,
                             int Hkv, int d, int bs, int64_t num_blocks, int64_t *slot_out,
                             int32_t *err_flag, void *stream) {
    if (B == 0 || n_new == 0) return PA_OK;
    if (!k_new || !v_new || !kq_cache || !vq_cache || !k_scale || !v_scale || !score_pool ||
        !block_tables || !positions || !err_flag)
        return PA_ERR_NULL;
    int rc = check_common(B, Hkv, d, bs, max_blocks_per_seq, num_blocks, block_stride);
    if (rc) return rc;
    if (n_new < 0) return PA_ERR_SHAPE;
    if (!al16(k_new) || !al16(v_new) || !al16(kq_cache) || !al16(vq_cache) || !al16(k_scale) ||
        !al16(v_scale) || block_stride % 16 != 0)
        return PA_ERR_ALIGN;
    const int sms = device_sms();
    if (sms < 0) return sms;
    pkv::AppendArgs a{block_tables, positions, slot_out, err_flag, block_stride, num_blocks,
                      B, n_new, Hkv, d, bs, max_blocks_per_seq};
    return finish(pkv::launch_append_int8(k_new, v_new, kq_cache, vq_cache, k_scale, v_scale,
                                          score_pool, a, sms, static_cast<cudaStream_t>(stream)));
}

int pe_select_evict_block_pooled(int32_t *evict, float *block_means, const float *score_pool,
                                 const int32_t *block_tables, int max_blocks_per_seq,
                                 const int32_t *ctx_lens, int B, int Hkv, int bs,
                                 int64_t num_blocks, int32_t *err_flag, void *stream) {
    if (B == 0) return PA_OK;
    if (!evict || !score_pool || !block_tables || !ctx_lens || !err_flag) return PA_ERR_NULL;
    if (B < 0 || B > 65535 || max_blocks_per_seq < 1 || Hkv < 1 || bs < 1 || num_blocks < 1)
        return PA_ERR_SHAPE;
    const int sms = device_sms();
    if (sms < 0) return sms;
    return finish(pkv::launch_select_pooled(evict, block_means, score_pool, block_tables,
                                            ctx_lens, err_flag, B, max_blocks_per_seq, Hkv, bs,
                                            num_blocks, static_cast<cudaStream_t>(stream)));
}

size_t pa_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int bs, int max_blocks_per_seq,
                                 int num_splits) {
    if (B <= 0 || Hq < 1 || Hkv < 1 || bs < 1 || max_blocks_per_seq < 1) return 0;
    const int sms = device_sms();
    if (sms < 0) return 0;
    if (Hq < Hkv || Hq % Hkv != 0 || (d != 64 && d != 128)) return 0;
    // one size serves pa_decode, pa_decode_int8 and pa_decode_fp8 alike
    size_t mx = 0;
    for (int kv = pkv::kKvBf16; kv <= pkv::kKvFp8; ++kv) {
        const size_t w = pkv::make_decode_plan(B, Hq, Hkv, d, bs, max_blocks_per_seq, num_splits,
                                               kv, sms).ws_total;
        mx = w > mx ? w : mx;
    }
    return mx;
}

int pa_decode_plan(int B, int Hq, int Hkv, int d, int bs, int max_blocks_per_seq, int num_splits,
                   int *num_splits_out, int *chunk_tokens_out, int *launches_out,
                   int *staged_out) {
    if (!num_splits_out || !chunk_tokens_out) return PA_ERR_NULL;
    if (B < 0 || Hq < 1 || Hkv < 1 || bs < 1 || max_blocks_per_seq < 1) return PA_ERR_SHAPE;
    if (d != 64 && d != 128) return PA_ERR_SHAPE;
    const int sms = device_sms();
    if (sms < 0) return sms;
    if (Hq < Hkv || Hq % Hkv != 0) return PA_ERR_SHAPE;
    const pkv::DecodePlan p =
        pkv::make_decode_plan(B, Hq, Hkv, d, bs, max_blocks_per_seq, num_splits, pkv::kKvBf16, sms);
    *num_splits_out = p.S;
    *chunk_tokens_out = p.chunk;
    if (launches_out)
        *launches_out = p.kernel == 1 ? 2 + ((p.S > 1 || p.wph > 1) ? 1 : 0) : 1 + (p.S > 1 ? 1 : 0);
    if (staged_out) *staged_out = p.kernel == 1 ? 1 : 0;
    return PA_OK;
}

int pa_decode(uint16_t *out, const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
              int64_t block_stride, const int32_t *block_tables, int max_blocks_per_seq,
              const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs, int64_t num_blocks,
              float scale, int num_splits, void *workspace, size_t workspace_bytes,
              int32_t *err_flag, void *stream) {
    return decode_entry(out, q, k_cache, v_cache, nullptr, nullptr, pkv::kKvBf16, block_stride,
                        block_tables, max_blocks_per_seq, ctx_lens, B, Hq, Hkv, d, bs, num_blocks,
                        scale, num_splits, workspace, workspace_bytes, err_flag, stream);
}

int pa_decode_int8(uint16_t *out, const uint16_t *q, const int8_t *kq_cache,
                   const int8_t *vq_cache, const float *k_scale, const float *v_scale,
                   int64_t block_stride, const int32_t *block_tables, int max_blocks_per_seq,
                   const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs,
                   int64_t num_blocks, float scale, int num_splits, void *workspace,
                   size_t workspace_bytes, int32_t *err_flag, void *stream) {
    return decode_entry(out, q, kq_cache, vq_cache, k_scale, v_scale, pkv::kKvInt8, block_stride,
                        block_tables, max_blocks_per_seq, ctx_lens, B, Hq, Hkv, d, bs, num_blocks,
                        scale, num_splits, workspace, workspace_bytes, err_flag, stream);
}

int pa_append_kv_fp8(const uint16_t *k_new, const uint16_t *v_new, uint8_t *k8_cache,
                     uint8_t *v8_cache, int64_t block_stride, const int32_t *block_tables,
                     int max_blocks_per_seq, const int32_t *positions, int B, int n_new, int Hkv,
                     int d, int bs, int64_t num_blocks, int64_t *slot_out, int32_t *err_flag,
                     void *stream) {
    if (B == 0 || n_new == 0) return PA_OK;
    if (!k_new || !v_new || !k8_cache || !v8_cache || !block_tables || !positions || !err_flag)
        return PA_ERR_NULL;
    int rc = check_common(B, Hkv, d, bs, max_blocks_per_seq, num_blocks, block_stride);
    if (rc) return rc;
    if (n_new < 0) return PA_ERR_SHAPE;
    if (!al16(k_new) || !al16(v_new) || !al16(k8_cache) || !al16(v8_cache) ||
        block_stride % 16 != 0)
        return PA_ERR_ALIGN;
    const int sms = device_sms();
    if (sms < 0) return sms;
    pkv::AppendArgs a{block_tables, positions, slot_out, err_flag, block_stride, num_blocks,
                      B, n_new, Hkv, d, bs, max_blocks_per_seq};
    return finish(pkv::launch_append_fp8(k_new, v_new, k8_cache, v8_cache, a, sms,
                                         static_cast<cudaStream_t>(stream)));
}

int pa_decode_fp8(uint16_t *out, const uint16_t *q, const uint8_t *k8_cache,
                  const uint8_t *v8_cache, int64_t block_stride, const int32_t *block_tables,
                  int max_blocks_per_seq, const int32_t *ctx_lens, int B, int Hq, int Hkv, int d,
                  int bs, int64_t num_blocks, float scale, int num_splits, void *workspace,
                  size_t workspace_bytes, int32_t *err_flag, void *stream) {
    return decode_entry(out, q, k8_cache, v8_cache, nullptr, nullptr, pkv::kKvFp8, block_stride,
                        block_tables, max_blocks_per_seq, ctx_lens, B, Hq, Hkv, d, bs, num_blocks,
                        scale, num_splits, workspace, workspace_bytes, err_flag, stream);
}

int pa_decode_prepare(const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs,
                      int max_blocks_per_seq, int num_splits, void *workspace,
                      size_t workspace_bytes, int32_t *err_flag, void *stream) {
    if (B == 0) return PA_OK;
    if (!ctx_lens || !err_flag) return PA_ERR_NULL;
    if (B < 0 || B > 65535 || Hkv < 1 || Hkv > 65535 || bs < 1 || max_blocks_per_seq < 1)
        return PA_ERR_SHAPE;
    if (d != 64 && d != 128) return PA_ERR_SHAPE;
    if ((int64_t)max_blocks_per_seq * bs > INT32_MAX) return PA_ERR_SHAPE;
    if (Hq < Hkv || Hq % Hkv != 0 || Hq / Hkv > 16) return PA_ERR_SHAPE;
    const int sms = device_sms();
    if (sms < 0) return sms;
    const pkv::DecodePlan plan =
        pkv::make_decode_plan(B, Hq, Hkv, d, bs, max_blocks_per_seq, num_splits, pkv::kKvBf16, sms);
    if (plan.kernel != 1) return PA_OK;  // the general-shape kernel keeps no device plan
    if (!workspace || workspace_bytes < plan.ws_total) return PA_ERR_WORKSPACE;
    if (!al16(workspace)) return PA_ERR_ALIGN;
    pkv::DecodeArgs a;
    memset(&a, 0, sizeof a);
    a.ctx_lens = ctx_lens;
    a.err = err_flag;
    a.ws = workspace;
    a.plan = plan;
    a.B = B;
    a.MB = max_blocks_per_seq;
    a.bs = bs;
    return finish(pkv::launch_decode_plan_only(a, static_cast<cudaStream_t>(stream)));
}

int pa_decode_planned(uint16_t *out, const uint16_t *q, const uint16_t *k_cache,
                      const uint16_t *v_cache, int64_t block_stride, const int32_t *block_tables,
                      int max_blocks_per_seq, const int32_t *ctx_lens, int B, int Hq, int Hkv,
                      int d, int bs, int64_t num_blocks, float scale, int num_splits,
                      void *workspace, size_t workspace_bytes, int32_t *err_flag, void *stream) {
    return decode_entry(out, q, k_cache, v_cache, nullptr, nullptr, pkv::kKvBf16, block_stride,
                        block_tables, max_blocks_per_seq, ctx_lens, B, Hq, Hkv, d, bs, num_blocks,
                        scale, num_splits, workspace, workspace_bytes, err_flag, stream, 1);
}

int pa_decode_select_pooled(uint16_t *out, const uint16_t *q, const uint16_t *k_cache,
                            const uint16_t *v_cache, int64_t block_stride,
                            const int32_t *block_tables, int max_blocks_per_seq,
                            const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs,
                            int64_t num_blocks, float scale, int num_splits, void *workspace,
                            size_t workspace_bytes, int32_t *evict, float *block_means,
                            const float *score_pool, int32_t *err_flag, void *stream) {
    if (B > 0 && (!evict || !score_pool)) return PA_ERR_NULL;
    return decode_entry(out, q, k_cache, v_cache, nullptr, nullptr, pkv::kKvBf16, block_stride,
                        block_tables, max_blocks_per_seq, ctx_lens, B, Hq, Hkv, d, bs, num_blocks,
                        scale, num_splits, workspace, workspace_bytes, err_flag, stream, 0, evict,
                        block_means, score_pool);
}

int pa_decode_planned_select_pooled(uint16_t *out, const uint16_t *q, const uint16_t *k_cache,
                                    const uint16_t *v_cache, int64_t block_stride,
                                    const int32_t *block_tables, int max_blocks_per_seq,
                                    const int32_t *ctx_lens, int B, int Hq, int Hkv, int d,
                                    int bs, int64_t num_blocks, float scale, int num_splits,
                                    void *workspace, size_t workspace_bytes, int32_t *evict,
                                    float *block_means, const float *score_pool,
                                    int32_t *err_flag, void *stream) {
    if (B > 0 && (!evict || !score_pool)) return PA_ERR_NULL;
    return decode_entry(out, q, k_cache, v_cache, nullptr, nullptr, pkv::kKvBf16, block_stride,
                        block_tables, max_blocks_per_seq, ctx_lens, B, Hq, Hkv, d, bs, num_blocks,
                        scale, num_splits, workspace, workspace_bytes, err_flag, stream, 1, evict,
                        block_means, score_pool);
}

int pa_decode_int8_planned(uint16_t *out, const uint16_t *q, const int8_t *kq_cache,
                           const int8_t *vq_cache, const float *k_scale, const float *v_scale,
                           int64_t block_stride, const int32_t *block_tables,
                           int max_blocks_per_seq, const int32_t *ctx_lens, int B, int Hq,
                           int Hkv, int d, int bs, int64_t num_blocks, float scale,
                           int num_splits, void *workspace, size_t workspace_bytes,
                           int32_t *err_flag, void *stream) {
    return decode_entry(out, q, kq_cache, vq_cache, k_scale, v_scale, pkv::kKvInt8, block_stride,
                        block_tables, max_blocks_per_seq, ctx_lens, B, Hq, Hkv, d, bs, num_blocks,
                        scale, num_splits, workspace, workspace_bytes, err_flag, stream, 1);
}

int pa_decode_fp8_planned(uint16_t *out, const uint16_t *q, const uint8_t *k8_cache,
                          const uint8_t *v8_cache, int64_t block_stride,
                          const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs,
                          int64_t num_blocks, float scale, int num_splits, void *workspace,
                          size_t workspace_bytes, int32_t *err_flag, void *stream) {
    return decode_entry(out, q, k8_cache, v8_cache, nullptr, nullptr, pkv::kKvFp8, block_stride,
                        block_tables, max_blocks_per_seq, ctx_lens, B, Hq, Hkv, d, bs, num_blocks,
                        scale, num_splits, workspace, workspace_bytes, err_flag, stream, 1);
}

int pe_score_tokens(float *scores, const uint16_t *k_cache, const uint16_t *v_cache,
                    int64_t block_stride, const int32_t *block_tables, int max_blocks_per_seq,
                    const int32_t *ctx_lens, int B, int Hkv, int d, int bs, int64_t num_blocks,
                    int32_t *err_flag, void *stream) {
    if (B == 0) return PA_OK;
    if (!scores || !k_cache || !v_cache || !block_tables || !ctx_lens || !err_flag)
        return PA_ERR_NULL;
    int rc = check_common(B, Hkv, d, bs, max_blocks_per_seq, num_blocks, block_stride);
    if (rc) return rc;
    if (!al16(k_cache) || !al16(v_cache) || (block_stride * 2) % 16 != 0) return PA_ERR_ALIGN;
    const int sms = device_sms();
    if (sms < 0) return sms;
    pkv::ScoreArgs a{scores, k_cache, v_cache, block_tables, ctx_lens, err_flag, block_stride,
                     num_blocks, B, Hkv, d, bs, max_blocks_per_seq};
    return finish(pkv::launch_score(a, static_cast<cudaStream_t>(stream)));
}

int pe_select_evict_block(int32_t *evict, float *block_means, const float *scores,
                          const int32_t *ctx_lens, int B, int max_blocks_per_seq, int Hkv, int bs,
                          void *stream) {
    if (B == 0) return PA_OK;
    if (!evict || !scores || !ctx_lens) return PA_ERR_NULL;
    if (B < 0 || max_blocks_per_seq < 1 || Hkv < 1 || bs < 1) return PA_ERR_SHAPE;
    const int sms = device_sms();
    if (sms < 0) return sms;
    return finish(pkv::launch_select_evict(evict, block_means, scores, ctx_lens, B,
                                           max_blocks_per_seq, Hkv, bs,
                                           static_cast<cudaStream_t>(stream)));
}

int pa_decode_static_scratch(uint16_t *out, const uint16_t *q, const uint16_t *k_cache,
                             const uint16_t *v_cache, int64_t block_stride,
                             const int32_t *block_tables, int max_blocks_per_seq,
                             const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs,
                             int64_t num_blocks, float scale, int num_splits, int32_t *err_flag,
                             void *stream) {
    if (B == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !ctx_lens || !err_flag)
        return PA_ERR_NULL;
    if (num_splits < 0) return PA_ERR_SHAPE;
    int rc = check_common(B, Hkv, d, bs, max_blocks_per_seq, num_blocks, block_stride);
    if (rc) return rc;
    if (Hq < Hkv || Hq % Hkv != 0 || Hq / Hkv > 16) return PA_ERR_SHAPE;
    if (!(scale == scale)) return PA_ERR_SHAPE;
    if (!al16(out) || !al16(q) || !al16(k_cache) || !al16(v_cache) || (block_stride * 2) % 16 != 0)
        return PA_ERR_ALIGN;
    const int sms = device_sms();
    if (sms < 0) return sms;
    const size_t cap = PA_STATIC_SCRATCH_BYTES;
    auto ws_for = [&](int s) {
        return pkv::make_decode_plan(B, Hq, Hkv, d, bs, max_blocks_per_seq, s, pkv::kKvBf16, sms)
            .ws_total;
    };
    int splits = num_splits;
    if (splits == 0 && ws_for(0) > cap) {
        // the automatic plan does not fit: the largest partition count whose scratch
        // fits (an explicit count; when the automatic plan fits, 0 is passed on and the
        // call partitions exactly as pa_decode does)
        int lo = 1, hi = pkv::make_decode_plan(B, Hq, Hkv, d, bs, max_blocks_per_seq, 0,
                                               pkv::kKvBf16, sms).S;
        if (hi < 1) hi = 1;
        while (lo < hi) {  // invariant: ws(lo) fits or lo == 1
            const int mid = (lo + hi + 1) / 2;
            if (ws_for(mid) <= cap)
                lo = mid;
            else
                hi = mid - 1;
        }
        splits = lo;
    }
    if (ws_for(splits) > cap) return PA_ERR_WORKSPACE;
    void *ws = static_scratch_address();
    if (!ws) return PA_ERR_CUDA;
    return decode_entry(out, q, k_cache, v_cache, nullptr, nullptr, pkv::kKvBf16, block_stride,
                        block_tables, max_blocks_per_seq, ctx_lens, B, Hq, Hkv, d, bs, num_blocks,
                        scale, splits, ws, cap, err_flag, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// PagedEviction prefill stage and table compaction
// ---------------------------------------------------------------------------
namespace {
int check_prefill_rows(const uint16_t *k, const uint16_t *v, int64_t T, int Hkv, int d) {
    if (!k || !v) return PA_ERR_NULL;
    if (T < 0 || Hkv < 1 || Hkv > 65535) return PA_ERR_SHAPE;
    if (d != 64 && d != 128 && d != 256) return PA_ERR_SHAPE;
    if (!al16(k) || !al16(v)) return PA_ERR_ALIGN;
    return PA_OK;
}
}  // namespace

int pe_prefill_scores(float *scores, const uint16_t *k, const uint16_t *v, int64_t T, int Hkv,
                      int d, void *stream) {
    if (T == 0) return PA_OK;
    if (!scores) return PA_ERR_NULL;
    int rc = check_prefill_rows(k, v, T, Hkv, d);
    if (rc) return rc;
    if ((T + 7) / 8 > INT32_MAX) return PA_ERR_SHAPE;
    const int sms = device_sms();
    if (sms < 0) return sms;
    return finish(pkv::launch_prefill_scores(scores, k, v, T, Hkv, d,
                                             static_cast<cudaStream_t>(stream)));
}

int pe_prefill_select(int32_t *keep_idx, int32_t *kept_len, const float *scores,
                      const int32_t *cu_seqlens, int B, int budget, int32_t *err_flag,
                      void *stream) {
    if (B == 0) return PA_OK;
    if (!keep_idx || !kept_len || !scores || !cu_seqlens || !err_flag) return PA_ERR_NULL;
    if (B < 0 || B > INT32_MAX / 2 || budget < 1) return PA_ERR_SHAPE;
    const int sms = device_sms();
    if (sms < 0) return sms;
    return finish(pkv::launch_prefill_select(keep_idx, kept_len, scores, cu_seqlens, B, budget,
                                             err_flag, static_cast<cudaStream_t>(stream)));
}

int pe_prefill_pack(uint16_t *k_cache, uint16_t *v_cache, int64_t block_stride,
                    const int32_t *block_tables, int max_blocks_per_seq, const uint16_t *k,
                    const uint16_t *v, const int32_t *cu_seqlens, const int32_t *keep_idx,
                    const int32_t *kept_len, int B, int budget, int Hkv, int d, int bs,
                    int64_t num_blocks, int32_t *err_flag, void *stream) {
    if (B == 0) return PA_OK;
    if (!k_cache || !v_cache || !block_tables || !cu_seqlens || !keep_idx || !kept_len ||
        !err_flag)
        return PA_ERR_NULL;
    int rc = check_prefill_rows(k, v, 1, Hkv, d);
    if (rc) return rc;
    if (B < 0 || budget < 1 || bs < 1 || max_blocks_per_seq < 1 || num_blocks < 1)
        return PA_ERR_SHAPE;
    if (block_stride < (int64_t)bs * Hkv * d) return PA_ERR_SHAPE;
    if ((int64_t)B * budget > (int64_t)INT32_MAX * 8) return PA_ERR_SHAPE;
    if (!al16(k_cache) || !al16(v_cache) || (block_stride * 2) % 16 != 0) return PA_ERR_ALIGN;
    const int sms = device_sms();
    if (sms < 0) return sms;
    return finish(pkv::launch_prefill_pack(k_cache, v_cache, block_stride, block_tables,
                                           max_blocks_per_seq, k, v, cu_seqlens, keep_idx,
                                           kept_len, B, budget, Hkv, d, bs, num_blocks, err_flag,
                                           static_cast<cudaStream_t>(stream)));
}

int pe_prefill_compress(uint16_t *k_cache, uint16_t *v_cache, int64_t block_stride,
                        const int32_t *block_tables, int max_blocks_per_seq, const uint16_t *k,
                        const uint16_t *v, const int32_t *cu_seqlens, int64_t T, int B,
                        int budget, int Hkv, int d, int bs, int64_t num_blocks, float *scores,
                        int32_t *keep_idx, int32_t *kept_len, int32_t *err_flag, void *stream) {
    if (B == 0) return PA_OK;
    // validate everything before the first launch
    if (!scores && T > 0) return PA_ERR_NULL;
    if (!k_cache || !v_cache || !block_tables || !cu_seqlens || !keep_idx || !kept_len ||
        !err_flag)
        return PA_ERR_NULL;
    int rc = check_prefill_rows(k, v, T, Hkv, d);
    if (rc) return rc;
    if (B < 0 || budget < 1 || bs < 1 || max_blocks_per_seq < 1 || num_blocks < 1)
        return PA_ERR_SHAPE;
    if (block_stride < (int64_t)bs * Hkv * d) return PA_ERR_SHAPE;
    if (!al16(k_cache) || !al16(v_cache) || (block_stride * 2) % 16 != 0) return PA_ERR_ALIGN;
    if (T > 0 && (rc = pe_prefill_scores(scores, k, v, T, Hkv, d, stream))) return rc;
    // T = 0 (every prompt empty): the select kernel keeps nothing and never reads
    // scores; a prompt longer than the budget would contradict T and is flagged
    if ((rc = finish(pkv::launch_prefill_select(keep_idx, kept_len, T > 0 ? scores : nullptr,
                                                cu_seqlens, B, budget, err_flag,
                                                static_cast<cudaStream_t>(stream)))))
        return rc;
    return pe_prefill_pack(k_cache, v_cache, block_stride, block_tables, max_blocks_per_seq, k, v,
                           cu_seqlens, keep_idx, kept_len, B, budget, Hkv, d, bs, num_blocks,
                           err_flag, stream);
}

int pe_evict_compact(int32_t *block_tables, int max_blocks_per_seq, int32_t *ctx_lens,
                     int32_t *freed, const int32_t *evict, int B, int bs, int32_t *err_flag,
                     void *stream) {
    if (B == 0) return PA_OK;
    if (!block_tables || !ctx_lens || !evict || !err_flag) return PA_ERR_NULL;
    if (B < 0 || max_blocks_per_seq < 1 || bs < 1) return PA_ERR_SHAPE;
    if ((int64_t)max_blocks_per_seq * bs > INT32_MAX) return PA_ERR_SHAPE;
    const int sms = device_sms();
    if (sms < 0) return sms;
    return finish(pkv::launch_evict_compact(block_tables, max_blocks_per_seq, ctx_lens, freed,
                                            evict, B, bs, err_flag,
                                            static_cast<cudaStream_t>(stream)));
}

int pe_select_evict_threshold(uint8_t *mask, int32_t *count, float *block_means,
                              const float *scores, const int32_t *ctx_lens, int B,
                              int max_blocks_per_seq, int Hkv, int bs, int64_t used_blocks,
                              int64_t total_blocks, double eviction_ratio,
                              double importance_threshold, void *stream) {
    if (B == 0) return PA_OK;
    if (!mask || !count || !scores || !ctx_lens) return PA_ERR_NULL;
    if (B < 0 || B > INT32_MAX / 2 || max_blocks_per_seq < 1 || Hkv < 1 || bs < 1)
        return PA_ERR_SHAPE;
    if (!(eviction_ratio >= 0.0 && eviction_ratio <= 1.0) ||
        importance_threshold != importance_threshold || used_blocks < 0 || total_blocks < 0)
        return PA_ERR_SHAPE;
    const int sms = device_sms();
    if (sms < 0) return sms;
    const int triggered = (double)used_blocks > (1.0 - eviction_ratio) * (double)total_blocks;
    return finish(pkv::launch_select_threshold(mask, count, block_means, scores, ctx_lens, B,
                                               max_blocks_per_seq, Hkv, bs, importance_threshold,
                                               triggered, static_cast<cudaStream_t>(stream)));
}

int pe_evict_compact_mask(int32_t *block_tables, int max_blocks_per_seq, int32_t *ctx_lens,
                          int32_t *freed, const uint8_t *mask, int B, int bs, int32_t *err_flag,
                          void *stream) {
    if (B == 0) return PA_OK;
    if (!block_tables || !ctx_lens || !mask || !err_flag) return PA_ERR_NULL;
    if (B < 0 || max_blocks_per_seq < 1 || bs < 1) return PA_ERR_SHAPE;
    if ((int64_t)max_blocks_per_seq * bs > INT32_MAX) return PA_ERR_SHAPE;
    const int sms = device_sms();
    if (sms < 0) return sms;
    return finish(pkv::launch_evict_compact_mask(block_tables, max_blocks_per_seq, ctx_lens, freed,
                                                 mask, B, bs, err_flag,
                                                 static_cast<cudaStream_t>(stream)));
}

size_t pa_prefill_attention_workspace_bytes(int B, int Hq, int Hkv, int d, int bs,
                                            int max_q_len) {
    if (B <= 0 || max_q_len <= 0 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || bs < 1) return 0;
    const int G = Hq / Hkv;
    if (G > 16 || (G & (G - 1)) != 0) return 0;
    const int sms = device_sms();
    if (sms < 0) return 0;
    pkv::PrefillAttnArgs a;
    memset(&a, 0, sizeof a);
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.G = G;
    a.d = d;
    a.bs = bs;
    return pkv::prefill_attn_tc_workspace_bytes(a, max_q_len, sms);
}

int pa_prefill_attention(uint16_t *out, const uint16_t *q, const int32_t *cu_q, int max_q_len,
                         const uint16_t *k_cache, const uint16_t *v_cache, int64_t block_stride,
                         const int32_t *block_tables, int max_blocks_per_seq,
                         const int32_t *ctx_lens, int B, int Hq, int Hkv, int d, int bs,
                         int64_t num_blocks, float scale, int32_t *err_flag, void *workspace,
                         size_t workspace_bytes, void *stream) {
    if (B == 0 || max_q_len == 0) return PA_OK;
    if (!out || !q || !cu_q || !k_cache || !v_cache || !block_tables || !ctx_lens || !err_flag)
        return PA_ERR_NULL;
    int rc = check_common(B, Hkv, d, bs, max_blocks_per_seq, num_blocks, block_stride);
    if (rc) return rc;
    if (max_q_len < 0 || Hq < Hkv || Hq % Hkv != 0) return PA_ERR_SHAPE;
    const int G = Hq / Hkv;
    if (G > 16 || (G & (G - 1)) != 0) return PA_ERR_SHAPE;
    if (!(scale == scale)) return PA_ERR_SHAPE;
    if ((int64_t)max_q_len * G / 64 + 1 > INT32_MAX) return PA_ERR_SHAPE;
    if (!al16(out) || !al16(q) || !al16(k_cache) || !al16(v_cache) || (block_stride * 2) % 16)
        return PA_ERR_ALIGN;
    if (workspace && !al16(workspace)) return PA_ERR_ALIGN;
    const int sms = device_sms();
    if (sms < 0) return sms;
    pkv::PrefillAttnArgs a;
    memset(&a, 0, sizeof a);
    a.out = out;
    a.q = q;
    a.cu_q = cu_q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_stride = block_stride;
    a.block_tables = block_tables;
    a.ctx_lens = ctx_lens;
    a.err = err_flag;
    a.N = num_blocks;
    a.B = B;
    a.MB = max_blocks_per_seq;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.G = G;
    a.d = d;
    a.bs = bs;
    a.scale_log2 = scale * 1.4426950408889634f;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // tcgen05 / TMEM kernel for d = 128 and 16-token-aligned blocks (TMA pages);
    // the mma.sync kernel covers every other supported shape
    return finish(pkv::prefill_attn_tc_supported(a)
                      ? pkv::launch_prefill_attn_tc(a, max_q_len, workspace, workspace_bytes, sms, st)
                      : pkv::launch_prefill_attn(a, max_q_len, st));
}

int pa_selftest_wait_timeout(int32_t *err_flag, void *stream) {
    if (!err_flag) return PA_ERR_NULL;
    const int sms = device_sms();
    if (sms < 0) return sms;
    return finish(pkv::launch_selftest_wait_timeout(err_flag, static_cast<cudaStream_t>(stream)));
}
