// decode_tc.cu -- paged decode attention for block sizes that are a multiple of
// 16: TMA-staged K/V tiles, bf16 tensor-core QK^T and PV, online softmax.
//
// Operator (ybb.press "LLM 推理 KV Cache 内存管理深度工程实践" §2.2 paged_attention_forward;
// t6page.pages.dev "KV cache", "PagedAttention 的算子"): for each sequence the K/V
// rows are found through the block table, and softmax(scale q.K) V is taken over
// the whole context; GQA (§6.2 of the first page): query head i reads kv head i/G.
//
// Work decomposition
//   A plan kernel (one CTA) reads the device context lengths and writes the
//   units (sequence, partition, token range) into the workspace.  The decode
//   kernel is persistent (one CTA per SM).
//   Automatic split: the contexts, laid end to end, are cut into one equal
//   token range per SM (at least 128 tokens); a cut inside a sequence snaps to
//   that sequence's 16-token tiles.  CTA i takes the pieces of range i, so every
//   SM reads the same number of K/V bytes whatever the mix of lengths.
//   Explicit split (num_splits > 0): every sequence is cut into near-equal
//   partitions of at most max_ctx / num_splits tokens, listed longest first, and
//   the producers take them from an atomic counter.
// Per CTA
//   warp 8 (producer): for each stage of 16*n_sub tokens (n_sub sub-tiles of 16
//   tokens; a stage carries about 64 KB of K and V), lane j looks the physical
//   block of sub-tile j up in the block table (through a 32-entry per-unit cache
//   held one id per lane) and issues 5-D TMA loads of the K and V rows of ALL kv
//   heads of those 16 tokens (one box per 128 bytes of d),
//   (INT8: plus bulk copies of the 16 tokens' K and V scale rows).
//   The tensor map orders the box as [head][token][64 elements] with 128-byte
//   swizzle, so each head's 16 token rows occupy 16 consecutive 128-byte rows
//   and ldmatrix reads them without bank conflicts.
//   warps 0..7 (consumers): warp w owns kv head w % Hkv and sub-tiles
//   w / Hkv + k * (8 / Hkv), k < tpw, of every stage; at a unit's start it loads
//   its query fragments
//   straight from global memory (L2).  S = Q K^T with the G query heads of the group as
//   the 16 rows of an m16n8k16 MMA (rows >= G are zero), online softmax on the
//   fp32 accumulators (exp2 domain), P split into two bf16 parts (hi + lo; for
//   G <= 8 the lo part fills the empty rows g + 8 of the same MMA), O += P V with
//   V read by ldmatrix.trans.  The stage is released to the producer through an mbarrier.
//   At a unit's last stage the warp writes either the normalised bf16 output
//   (single-partition sequence) or its (O, m, l) partial for the merge kernel.
// Masking: tokens at or past the unit's end get -inf logits, and their V rows
// are zeroed in registers, so stale or NaN data in unused slots never reaches
// the result.  Out-of-range block ids are not loaded; the sub-tile is skipped
// and PA_DEV_BAD_BLOCK is raised.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <utility>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "select_pooled.cuh"

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
    const float *k_scale;  // INT8 pools: [N][bs][Hkv] fp32
    const float *v_scale;
    int64_t N;
    int B, Hq, Hkv, G, bs, MB, S, nstage, stage_bytes, v_off, ks_off, vs_off, box_bytes;
    int wph;        // consumer warps per kv head (8 / Hkv): partial slots per unit
    int tpw;        // 16-token sub-tiles per warp per stage
    int n_sub;      // sub-tiles per stage (wph * tpw)
    int tpb_shift;  // log2(bs / 16) when bs / 16 is a power of two, else -1
    float scale_log2;
    unsigned long long sig;  // signature of the sizes; must match the plan's (header)
    const int32_t *cta_off;  // balanced plan: CTA i takes units cta_off[i] .. cta_off[i+1]-1
    const int4 *cta_first;   // balanced plan: a copy of CTA i's first unit
    int balanced;
    // the merge launch's first sel_ctas CTAs (0 or B) run the pooled block selection
    int sel_ctas;
    int32_t *sel_evict;
    float *sel_means;
    const float *sel_scores;
};

// ---------------------------------------------------------------------------
// plan: one CTA of 1024 threads
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t *ctx_lens, int32_t *err,
                                                   TcHeader *hdr, int32_t *ns, int4 *units, int B,
                                                   int max_ctx, int min_chunk, int target_units,
                                                   unsigned long long sig) {
    constexpr int kSerialParts = 32, kMaxLong = 256;
    __shared__ long long s_red[32];
    __shared__ int hist[1024];
    __shared__ int s_chunk, s_nlong;
    __shared__ int s_long[kMaxLong];
    const int tid = threadIdx.x;
    // launched programmatically after the previous kernel (e.g. the KV append):
    // let the decode kernel's CTAs get resident, then wait for the predecessor
    ptx::grid_launch_dependents();
    ptx::grid_dependency_wait();
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
        s_nlong = 0;
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
    // a thread per sequence (all lengths loaded at once); a sequence with more than
    // kSerialParts partitions is left to a warp whose lanes take its partitions, so a
    // few very long sequences do not serialise on a few threads
    const int warp = tid >> 5, lane = tid & 31, nwarps = (int)(blockDim.x >> 5);
    for (int b = tid; b < B; b += blockDim.x) {
        int len = ctx_lens[b];
        if (len < 0 || len > max_ctx) len = 0;
        int n, step;
        part(len, n, step);
        ns[b] = n;
        const int k = n > kSerialParts ? atomicAdd(&s_nlong, 1) : kMaxLong;
        if (k < kMaxLong) {
            s_long[k] = b;
        } else {
            for (int c = 0; c < n; ++c)
                atomicAdd(&hist[min(1023, min(step, len - c * step) / kTile)], 1);
        }
    }
    __syncthreads();
    const int nlong = min(s_nlong, kMaxLong);
    for (int k = warp; k < nlong; k += nwarps) {
        const int b = s_long[k];
        int len = ctx_lens[b];
        if (len < 0 || len > max_ctx) len = 0;
        int n, step;
        part(len, n, step);
        for (int c = lane; c < n; c += 32)
            atomicAdd(&hist[min(1023, min(step, len - c * step) / kTile)], 1);
    }
    __syncthreads();
    {   // exclusive prefix over the buckets, largest first (thread t owns bucket 1023 - t)
        const int k = 1023 - tid;
        const int v = hist[k];
        int inc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(kFull, inc, o);
            if ((tid & 31) >= o) inc += n;
        }
        __shared__ int s_warp[32];
        if ((tid & 31) == 31) s_warp[tid >> 5] = inc;
        __syncthreads();
        if (tid < 32) {
            int w = s_warp[tid];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(kFull, w, o);
                if (tid >= o) w += n;
            }
            s_warp[tid] = w;  // inclusive totals of warps 0..tid
        }
        __syncthreads();
        const int before = (tid >> 5) ? s_warp[(tid >> 5) - 1] : 0;
        hist[k] = before + inc - v;
        if (tid == 1023) {
            hdr->n_units = before + inc;
            hdr->counter = 0u;
            hdr->done = 0u;
            hdr->sig = sig;
        }
    }
    __syncthreads();
    for (int b = tid; b < B; b += blockDim.x) {
        int len = ctx_lens[b];
        if (len < 0 || len > max_ctx) len = 0;
        int n, step;
        part(len, n, step);
        if (n > kSerialParts && nlong > 0) {   // listed (unless the list overflowed)?
            bool listed = false;
            for (int k = 0; k < nlong && !listed; ++k) listed = s_long[k] == b;
            if (listed) continue;
        }
        for (int c = 0; c < n; ++c) {
            const int t0 = c * step, t1 = min(len, t0 + step);
            const int pos = atomicAdd(&hist[min(1023, (t1 - t0) / kTile)], 1);
            units[pos] = make_int4(b, c, t0, t1);
        }
    }
    for (int k = warp; k < nlong; k += nwarps) {
        const int b = s_long[k];
        int len = ctx_lens[b];
        if (len < 0 || len > max_ctx) len = 0;
        int n, step;
        part(len, n, step);
        for (int c = lane; c < n; c += 32) {
            const int t0 = c * step, t1 = min(len, t0 + step);
            const int pos = atomicAdd(&hist[min(1023, (t1 - t0) / kTile)], 1);
            units[pos] = make_int4(b, c, t0, t1);
        }
    }
}

// Exclusive prefix sum over the 1024 threads of a CTA (64-bit); *total gets the sum.
__device__ __forceinline__ long long cta_scan64(long long v, long long *total) {
    __shared__ long long s_w[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(kFull, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) s_w[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        long long x = s_w[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(kFull, x, o);
            if (lane >= o) x += y;
        }
        s_w[lane] = x;   // inclusive totals of warps 0..lane
    }
    __syncthreads();
    const long long before = warp ? s_w[warp - 1] : 0;
    *total = s_w[31];
    __syncthreads();
    return before + inc - v;
}

// ---------------------------------------------------------------------------
// balanced plan (automatic split): one CTA of 1024 threads.
// The contexts, laid end to end (T tokens), are cut into nr equal ranges of
// `range` = max(16-token multiple of ceil(T / P), min_chunk) tokens, one per decode
// CTA (nr <= P).  A cut that falls inside a sequence is snapped to the nearest
// 16-token tile boundary of that sequence, so every piece starts on a tile.  A
// range's pieces (its parts of consecutive sequences) go to its CTA; piece c of
// sequence b is partition c of b (ns[b] pieces; a sequence of length 0 has none
// and the merge writes its zero row).
// ---------------------------------------------------------------------------
constexpr int kMaxRanges = 1024;
constexpr int kSeqCache = 1024;   // sequences whose length and start stay in shared memory

__global__ void __launch_bounds__(1024) plan_balanced_kernel(
    const int32_t *ctx_lens, int32_t *err, TcHeader *hdr, int32_t *ns, int4 *units,
    int32_t *cta_off, int4 *cta_first, long long *starts, int B, int max_ctx, int min_chunk,
    int P, unsigned long long sig) {
    __shared__ int s_cnt[kMaxRanges];          // pieces per range, then fill positions
    __shared__ int s_off[kMaxRanges];          // first unit of each range
    __shared__ int s_len[kSeqCache];           // lengths and starts of sequences < kSeqCache
    __shared__ long long s_st[kSeqCache];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < kMaxRanges; i += 1024) s_cnt[i] = 0;   // (read only after barriers)
    ptx::grid_launch_dependents();
    ptx::grid_dependency_wait();
    auto clamp_len = [&](int b, bool flag) {
        int len = ctx_lens[b];
        if (len < 0 || len > max_ctx) {
            if (flag) raise_flag(err, PA_DEV_BAD_LEN);
            len = 0;
        }
        return len;
    };
    // ---- sequence starts (exclusive prefix sums of the lengths): kept in shared
    // memory for the first kSeqCache sequences, in the workspace for all
    long long run = 0;
    for (int b0 = 0; b0 < B; b0 += 1024) {
        const int b = b0 + tid;
        const int len = b < B ? clamp_len(b, true) : 0;
        long long tot;
        const long long st = run + cta_scan64(len, &tot);
        if (b < B) starts[b] = st;
        if (b < kSeqCache) {
            s_len[b] = len;
            s_st[b] = st;
        }
        run += tot;
    }
    // every thread derives the range and the number of ranges from the total
    const long long T = run;
    long long range = (T + P - 1) / P;
    range = (range + kTile - 1) / kTile * kTile;
    if (range < min_chunk) range = min_chunk;
    const int nr = T > 0 ? (int)((T + range - 1) / range) : 0;
    __syncthreads();   // publishes s_len / s_st and the workspace starts
    auto seq = [&](int b, int &len, long long &st) {
        if (b < kSeqCache) {
            len = s_len[b];
            st = s_st[b];
        } else {
            len = clamp_len(b, false);
            st = starts[b];
        }
    };
    // The candidate cuts of a sequence, i0 <= i < i1: the range boundaries i * range
    // strictly inside it; cut i lands on the sequence's nearest 16-token tile boundary
    // (at most its end).  A cut strictly inside the sequence starts a piece owned by
    // range i; the first piece belongs to the range holding the sequence's start:
    // i0 - 1, or i0 when cut i0 snaps onto the start (every earlier cut lies at or
    // before it, every later one after it).
    auto cand = [&](int len, long long st, int &i0, int &i1) {
        i0 = (int)(st / range) + 1;
        const long long e = (st + len - 1) / range + 1;
        i1 = (int)(e < nr ? e : nr);
    };
    auto cut = [&](int i, int len, long long st) {
        const long long o = (long long)i * range - st;   // 0 < o < len
        long long sn = (o + kTile / 2) / kTile * kTile;
        if (sn >= len) sn = len;
        return st + sn;
    };
    // Few sequences (B < 32, where one can hold many cuts): a warp takes a sequence
    // (b = warp, warp + 32, ...) and its lanes the candidate cuts.  Otherwise a thread
    // takes a sequence and walks its (few) candidates.
    const bool lanes = B < 32;
    const int grp = lanes ? lane : 0, gw = lanes ? 32 : 1;      // lane in the group, width
    const int g0 = lanes ? warp : tid, gstep = lanes ? 32 : 1024;  // first sequence, stride
    // ---- partitions per sequence and pieces per range, in one pass
    for (int b = g0; b < B; b += gstep) {
        int len, i0, i1;
        long long st;
        seq(b, len, st);
        int n = 0;
        if (len > 0) {
            cand(len, st, i0, i1);
            for (int i = i0 + grp; i < i1; i += gw) {
                const long long r = cut(i, len, st);
                if (r > st && r < st + len) {
                    ++n;
                    atomicAdd(&s_cnt[i], 1);
                }
            }
            n = 1 + (lanes ? __reduce_add_sync(kFull, n) : n);
            if (grp == 0) atomicAdd(&s_cnt[(i0 < i1 && cut(i0, len, st) == st) ? i0 : i0 - 1], 1);
        }
        if (grp == 0) ns[b] = n;
    }
    __syncthreads();
    // ---- per-range unit offsets (exclusive scan over the ranges; ranges >= nr empty)
    {
        long long tot;
        const int c = tid < nr ? s_cnt[tid] : 0;
        const long long off = cta_scan64(c, &tot);
        if (tid <= P) cta_off[tid] = (int)(tid < nr ? off : tot);
        if (tid < nr) s_cnt[tid] = s_off[tid] = (int)off;   // fill position of range tid
        if (tid == 0) {
            hdr->n_units = (int)tot;
            hdr->chunk = (int)min(range, (long long)INT32_MAX);
            hdr->counter = 0u;
            hdr->done = 0u;
            hdr->sig = sig;
        }
    }
    __syncthreads();
    // ---- the pieces: sequence b's valid cuts in order give partitions c = 1, 2, ...
    // (a warp per sequence: lane order, a carry counting the valid cuts of earlier
    // 32-candidate chunks); the unit placed first in a range is also copied to that
    // CTA's cta_first
    auto place = [&](int own, int4 u) {
        const int pos = atomicAdd(&s_cnt[own], 1);
        units[pos] = u;
        if (pos == s_off[own]) cta_first[own] = u;
    };
    for (int b = g0; b < B && !lanes; b += gstep) {   // a thread per sequence
        int len, i0, i1;
        long long st;
        seq(b, len, st);
        if (len == 0) continue;
        cand(len, st, i0, i1);
        const long long end = st + len;
        int own = (i0 < i1 && cut(i0, len, st) == st) ? i0 : i0 - 1, c = 0;
        long long t0 = st;
        for (int i = i0; i <= i1; ++i) {   // each valid cut ends a piece; the end, the last
            const long long r = i < i1 ? cut(i, len, st) : end;
            const bool is_cut = i < i1 && r > st && r < end;
            if (i < i1 && !is_cut) continue;
            const long long t1 = is_cut ? r : end;
            place(own, make_int4(b, c, (int)(t0 - st), (int)(t1 - st)));
            own = i;
            t0 = t1;
            ++c;
        }
    }
    for (int b = warp; b < B && lanes; b += 32) {   // a warp per sequence
        int len, i0, i1;
        long long st;
        seq(b, len, st);
        if (len == 0) continue;
        cand(len, st, i0, i1);
        const long long end = st + len;
        auto valid = [&](long long r) { return r > st && r < end; };
        int carry = 0;
        long long first_cut = end;   // where piece 0 ends
        for (int k0 = i0; k0 < i1; k0 += 32) {
            const int i = k0 + lane;
            const long long r = i < i1 ? cut(i, len, st) : end;
            const bool v = i < i1 && valid(r);
            const unsigned m = __ballot_sync(kFull, v);
            if (first_cut == end && m) first_cut = __shfl_sync(kFull, r, __ffs(m) - 1);
            if (v) {
                int j = i + 1;   // the next valid cut (only a sequence's last candidate
                long long rj = end;   // can be invalid, so this is short)
                for (; j < i1; ++j) {
                    rj = cut(j, len, st);
                    if (valid(rj)) break;
                }
                const long long t1 = j < i1 ? rj : end;
                const int c = 1 + carry + __popc(m & ((1u << lane) - 1u));
                place(i, make_int4(b, c, (int)(r - st), (int)(t1 - st)));
            }
            carry += __popc(m);
        }
        if (lane == 0)
            place((i0 < i1 && cut(i0, len, st) == st) ? i0 : i0 - 1,
                  make_int4(b, 0, 0, (int)(first_cut - st)));
    }
}

// ---------------------------------------------------------------------------
// decode: persistent, warp-specialised
// ---------------------------------------------------------------------------
template <int D, int KV>
__device__ __forceinline__ void producer(const CUtensorMap *kmap, const CUtensorMap *vmap,
                                         const Args &a, uint8_t *stages, StageMeta *meta,
                                         uint64_t *full, uint64_t *empty) {
    // one box covers 128 bytes of d: 64 bf16 or 128 one-byte (int8, e4m3) values
    constexpr bool I8 = KV == kKvInt8;
    constexpr int DC = KV != kKvBf16 ? D / 128 : D / 64;
    const int lane = threadIdx.x & 31;
    const int T_s = kTile * a.n_sub;
    const uint32_t sc_bytes = (uint32_t)kTile * a.Hkv * 4;  // one sub-tile's scale rows
    const uint32_t sub_bytes = 2u * DC * (uint32_t)a.box_bytes + (I8 ? 2u * sc_bytes : 0u);
    const int tpb = a.bs / kTile;                            // 16-token tiles per block
    // The header, this CTA's unit offsets and its first unit's copy are independent
    // loads issued together, one round trip before the first block-table lookup (the
    // offset and copy regions exist in every plan layout; an explicit plan ignores them).
    const unsigned long long hsig = a.hdr->sig;
    const int h_units = a.hdr->n_units;
    const int off0 = a.cta_off[blockIdx.x], off1 = a.cta_off[blockIdx.x + 1];
    const int4 un_first = a.cta_first[blockIdx.x];
    // a plan made for other sizes (a kept plan that does not match this call) is
    // not used: no unit is taken and the call flags it
    const bool plan_ok = hsig == a.sig;
    // balanced plan: this CTA's own list of units; otherwise all units, longest first,
    // taken from the counter
    const int u_first = plan_ok && a.balanced ? off0 : 0;
    const int n_units = !plan_ok ? 0 : a.balanced ? off1 : h_units;
    int u_next = u_first;
    if (!plan_ok && lane == 0 && blockIdx.x == 0) raise_flag(a.err, PA_DEV_BAD_PLAN);
    const uint64_t policy = ptx::policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = plan_ok;
    while (ok) {
        unsigned u = 0;
        if (a.balanced) {
            u = (unsigned)u_next++;
        } else {
            if (lane == 0) u = atomicAdd(&a.hdr->counter, 1u);
            u = __shfl_sync(kFull, u, 0);
        }
        if ((int)u >= n_units) break;
        const int4 un = (a.balanced && (int)u == u_first) ? un_first : a.units[u];
        const int b = un.x, c = un.y, t0 = un.z, t1 = un.w;
        const bool direct = (a.wph == 1) && (a.ns[b] == 1);
        const int nst = t1 > t0 ? (t1 - t0 + T_s - 1) / T_s : 1;
        const int32_t *bt_row = a.bt + (int64_t)b * a.MB;
        // lane k caches the physical id of block cache_base + k (blocks of this unit only)
        const int last_blk = t1 > t0 ? (t1 - 1) / a.bs : 0;
        int cache_base = 0x7fffffff, cache = -1;
        int ti = t0 / kTile;  // 16-token tile index of this lane's sub-tile, stage 0
        ti += lane;
        for (int si = 0; si < nst; ++si, ti += a.n_sub) {
            const int ts = t0 + si * T_s, te = min(ts + T_s, t1);
            // sub-tile of lane j (j < n_sub): tokens ts + 16 j .. ; its block and slot
            const int blk = a.tpb_shift >= 0 ? (ti >> a.tpb_shift) : ti / tpb;
            const int slot = (ti - blk * tpb) * kTile;
            const bool mine = lane < a.n_sub && ts + kTile * lane < te;
            const int blk_hi = __shfl_sync(kFull, blk, min(a.n_sub, 32) - 1);
            if (blk_hi - cache_base >= 32 || cache_base == 0x7fffffff) {  // (re)fill the cache
                cache_base = __shfl_sync(kFull, blk, 0);
                const int bk = cache_base + lane;
                cache = bk <= last_blk ? __ldg(bt_row + bk) : -1;
            }
            const int phys = __shfl_sync(kFull, cache, (blk - cache_base) & 31);
            const bool valid = mine && phys >= 0 && (int64_t)phys < a.N;
            const unsigned vmask = __ballot_sync(kFull, valid);
            const unsigned bad = __ballot_sync(kFull, mine && !valid);
            if (!ptx::mbar_wait(&empty[stage], phase ^ 1u)) {
                if (lane == 0) raise_flag(a.err, PA_DEV_TIMEOUT);
                ok = false;
                break;
            }
            uint8_t *sb = stages + (size_t)stage * a.stage_bytes;
            if (lane == 0) {
                StageMeta &m = meta[stage];
                m.b = b;
                m.c = c;
                m.ts = ts;
                m.te = te;
                m.bad = (int)bad;
                m.flags = (si == 0 ? kFirst : 0) | (si == nst - 1 ? kLast : 0) |
                          (direct ? kDirect : 0);
                if (bad) raise_flag(a.err, PA_DEV_BAD_BLOCK);
                ptx::mbar_arrive_expect_tx(&full[stage], __popc(vmask) * sub_bytes);
            }
            __syncwarp();
            if (valid) {  // each lane loads its own sub-tile
#pragma unroll
                for (int dc = 0; dc < DC; ++dc) {
                    const size_t off = (size_t)(lane * DC + dc) * a.box_bytes;
                    ptx::tma_load_5d_hint(sb + off, kmap, &full[stage], 0, slot, 0, dc, phys,
                                          policy);
                    ptx::tma_load_5d_hint(sb + a.v_off + off, vmap, &full[stage], 0, slot, 0, dc,
                                          phys, policy);
                }
                if (I8) {
                    const int64_t srow = ((int64_t)phys * a.bs + slot) * a.Hkv;
                    ptx::bulk_load(sb + a.ks_off + lane * sc_bytes, a.k_scale + srow, sc_bytes,
                                   &full[stage]);
                    ptx::bulk_load(sb + a.vs_off + lane * sc_bytes, a.v_scale + srow, sc_bytes,
                                   &full[stage]);
                }
            }
            if (++stage == a.nstage) {
                stage = 0;
                phase ^= 1u;
            }
        }
    }
    if (ok || !plan_ok) {
        if (ptx::mbar_wait(&empty[stage], phase ^ 1u)) {
            if (lane == 0) {
                meta[stage].flags = kEnd;
                ptx::mbar_arrive(&full[stage]);
            }
        } else if (lane == 0) {
            raise_flag(a.err, PA_DEV_TIMEOUT);
        }
    }
    // this CTA takes no more units: the last CTA to get here resets the unit counter
    // (every CTA's last fetch came before its increment), so the plan can serve the
    // next decode call without the plan kernel
    if (lane == 0 && plan_ok) {
        __threadfence();
        if (atomicAdd(&a.hdr->done, 1u) == gridDim.x - 1) {
            atomicExch(&a.hdr->counter, 0u);
            atomicExch(&a.hdr->done, 0u);
        }
    }
}

// Load the query fragments of rows g (and g + 8) of kv head h for sequence b
// straight from global memory (L2): k-step kk of thread (g, tig) takes dims
// 16*kk + 2*tig (+1) and 16*kk + 8 + 2*tig (+1), the A-operand layout of the
// m16n8k16 MMA.  Rows >= G are zero.
template <int D, bool G16>
__device__ __forceinline__ void load_q_bf16(const Args &a, int b, int h, int g, int tig,
                                            uint32_t (&qa)[D / 16][2],
                                            uint32_t (&qb)[G16 ? D / 16 : 1][2]) {
    const int row = h * a.G + g;
    const uint32_t *qr =
        reinterpret_cast<const uint32_t *>(a.q + ((int64_t)b * a.Hq + row) * D) + tig;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        qa[kk][0] = g < a.G ? __ldg(qr + kk * 8) : 0u;
        qa[kk][1] = g < a.G ? __ldg(qr + kk * 8 + 4) : 0u;
        if constexpr (G16) {
            qb[kk][0] = g + 8 < a.G ? __ldg(qr + 4 * D + kk * 8) : 0u;
            qb[kk][1] = g + 8 < a.G ? __ldg(qr + 4 * D + kk * 8 + 4) : 0u;
        }
    }
}

// Low bf16 part of the pair (x, y) whose high parts are packed in `hi`:
// bf16(x - hi.x), bf16(y - hi.y); the differences are exact in fp32.
// 2^x on the MUFU pipe (ex2.approx.ftz: relative error ~2^-22, far inside the bf16 /
// fp16 weights it feeds; 2^-inf = 0), for the consumers' softmax weights.
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t bf16_lo_part(float x, float y, uint32_t hi) {
    return ptx::pack_bf16(x - bf16_lo(hi), y - bf16_hi(hi));
}

// The sequence of this CTA's first unit (balanced plan: its copy sits beside the
// CTA's offsets), or -1.  The consumers load that unit's query before its first stage
// lands, so the query's round trip overlaps the first K/V loads instead of following
// them.  A CTA without units (or a refused plan) may read a stale copy: any sequence
// in range is only a wasted load, the query is reloaded for every other unit.
__device__ __forceinline__ int first_unit_seq(const Args &a) {
    if (!a.balanced) return -1;
    const int b = a.cta_first[blockIdx.x].x;
    return (b >= 0 && b < a.B) ? b : -1;
}

template <int D, bool G16>
__device__ __forceinline__ void consumer(const Args &a, uint8_t *stages, StageMeta *meta,
                                         uint64_t *full, uint64_t *empty) {
    constexpr int DC = D / 64;
    constexpr int KS = D / 16;  // k-steps of QK^T (and n-tile pairs of PV)
    constexpr int NT = D / 8;   // n-tiles of the output
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = warp % a.Hkv, jw = warp / a.Hkv;
    const int g = lane >> 2, tig = lane & 3;
    const int mi = lane >> 3, ri = lane & 7;
    // per-lane byte offsets inside a (head, sub-tile, 64-element) box
    const int tk = ri + ((mi >> 1) << 3);        // K: matrices 0,1 -> tokens 0-7; 2,3 -> 8-15
    const int ck = mi & 1;                       //    matrices 1,3 -> second 16-byte chunk
    const int tv = ri + ((mi & 1) << 3);         // V: matrices 0,2 -> tokens 0-7; 1,3 -> 8-15
    const int cv = mi >> 1;
    const uint32_t stage0 = ptx::smem_u32(stages);
    // sub-tile jj of a stage: box (jj * DC + dc); head h at row h * 16 + token
    const uint32_t head_off = (uint32_t)(h * kTile * kBoxRow);
    const uint32_t sub_bytes = (uint32_t)(DC * a.box_bytes);
    const uint32_t dc_bytes = (uint32_t)a.box_bytes;

    uint32_t qa[KS][2];
    uint32_t qb[G16 ? KS : 1][2];
    float o[NT][2];
    float ob[G16 ? NT : 1][2];
    float m = -INFINITY, l = 0.f, mb = -INFINITY, lb = 0.f;
    // (d = 128 only: on the d = 64 shape the early load measured slower, 19.63 ->
    // 19.86 us per c2 call, where d = 128 calls gained 0.8-1 %)
    int q_b = D == 128 ? first_unit_seq(a) : -1;   // the sequence whose query the registers hold
    if (q_b >= 0) load_q_bf16<D, G16>(a, q_b, h, g, tig, qa, qb);
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
            if (mt.b != q_b) load_q_bf16<D, G16>(a, mt.b, h, g, tig, qa, qb);
            q_b = -1;
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
        for (int k = 0; k < a.tpw; ++k) {
        const int jj = jw + a.wph * k;  // this warp's k-th sub-tile of the stage
        const int tj = mt.ts + kTile * jj;
        const int nv = max(0, min(kTile, mt.te - tj));
        if (nv > 0 && !((mt.bad >> jj) & 1)) {
            const uint32_t kbase = sb + jj * sub_bytes + head_off;
            const uint32_t vbase = sb + a.v_off + jj * sub_bytes + head_off;
            // ---- S = Q K^T : two n-tiles of 8 tokens; even/odd k-steps in separate
            // accumulators to halve the dependent MMA chain
            float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
            float e0[4] = {0.f, 0.f, 0.f, 0.f}, e1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                const int dc = kk >> 2, c = ((kk & 3) << 1) + ck;
                uint32_t r[4];
                ptx::ldmatrix_x4(r, kbase + dc * dc_bytes + tk * kBoxRow + ((c ^ ri) << 4));
                float(&x0)[4] = (kk & 1) ? e0 : s0;
                float(&x1)[4] = (kk & 1) ? e1 : s1;
                if constexpr (G16) {
                    ptx::mma_bf16(x0, qa[kk][0], qb[kk][0], qa[kk][1], qb[kk][1], r[0], r[1]);
                    ptx::mma_bf16(x1, qa[kk][0], qb[kk][0], qa[kk][1], qb[kk][1], r[2], r[3]);
                } else {
                    ptx::mma_bf16(x0, qa[kk][0], 0u, qa[kk][1], 0u, r[0], r[1]);
                    ptx::mma_bf16(x1, qa[kk][0], 0u, qa[kk][1], 0u, r[2], r[3]);
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                s0[i] += e0[i];
                s1[i] += e1[i];
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
            const float alpha = ex2_fast(m - mu);
            const float p0 = ex2_fast(x0 - mu), p1 = ex2_fast(x1 - mu);
            const float p2 = ex2_fast(x2 - mu), p3 = ex2_fast(x3 - mu);
            l = l * alpha + ((p0 + p1) + (p2 + p3));
            m = mn;
            // P = hi + lo, both bf16: p - hi is exact in fp32 and lo carries the 8 bits
            // that one bf16 would drop (a single bf16 P can be off by 2^-9 of the weight,
            // too coarse when a few tokens hold most of the weight).  For G <= 8 the lo
            // parts ride in the otherwise empty rows g + 8 of the same MMA.
            const uint32_t pa0 = ptx::pack_bf16(p0, p1), pa2 = ptx::pack_bf16(p2, p3);
            uint32_t pa1 = bf16_lo_part(p0, p1, pa0), pa3 = bf16_lo_part(p2, p3, pa2);
            uint32_t la0 = 0u, la1 = 0u, la2 = 0u, la3 = 0u;
            float alphab = 1.f;
            if constexpr (G16) {
                la0 = pa1;
                la2 = pa3;
                float y0 = va0 ? s0[2] * sl : -INFINITY, y1 = va1 ? s0[3] * sl : -INFINITY;
                float y2 = vb0 ? s1[2] * sl : -INFINITY, y3 = vb1 ? s1[3] * sl : -INFINITY;
                float my = fmaxf(fmaxf(y0, y1), fmaxf(y2, y3));
                my = fmaxf(my, __shfl_xor_sync(kFull, my, 1));
                my = fmaxf(my, __shfl_xor_sync(kFull, my, 2));
                const float mnb = fmaxf(mb, my);
                const float mub = mnb == -INFINITY ? 0.f : mnb;
                alphab = ex2_fast(mb - mub);
                const float q0 = ex2_fast(y0 - mub), q1 = ex2_fast(y1 - mub);
                const float q2 = ex2_fast(y2 - mub), q3 = ex2_fast(y3 - mub);
                lb = lb * alphab + ((q0 + q1) + (q2 + q3));
                mb = mnb;
                pa1 = ptx::pack_bf16(q0, q1);
                pa3 = ptx::pack_bf16(q2, q3);
                la1 = bf16_lo_part(q0, q1, pa1);
                la3 = bf16_lo_part(q2, q3, pa3);
            }
            // rescale only when some row maximum moved (alpha == 1 exactly otherwise)
            if (__any_sync(kFull, alpha != 1.f || alphab != 1.f)) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    o[nt][0] *= alpha;
                    o[nt][1] *= alpha;
                    if constexpr (G16) {
                        ob[nt][0] *= alphab;
                        ob[nt][1] *= alphab;
                    }
                }
            }
            // ---- O += P V
            const uint32_t mlo = (va0 ? 0x0000ffffu : 0u) | (va1 ? 0xffff0000u : 0u);
            const uint32_t mhi = (vb0 ? 0x0000ffffu : 0u) | (vb1 ? 0xffff0000u : 0u);
            const bool partial = nv < kTile;
#pragma unroll
            for (int pj = 0; pj < KS; ++pj) {
                const int dc = pj >> 2, c = ((pj & 3) << 1) + cv;
                uint32_t r[4];
                ptx::ldmatrix_x4_trans(r, vbase + dc * dc_bytes + tv * kBoxRow + ((c ^ ri) << 4));
                if (partial) {
                    r[0] &= mlo;
                    r[1] &= mhi;
                    r[2] &= mlo;
                    r[3] &= mhi;
                }
                float d0[4] = {o[2 * pj][0], o[2 * pj][1], 0.f, 0.f};
                float d1[4] = {o[2 * pj + 1][0], o[2 * pj + 1][1], 0.f, 0.f};
                if constexpr (G16) {
                    d0[2] = ob[2 * pj][0];
                    d0[3] = ob[2 * pj][1];
                    d1[2] = ob[2 * pj + 1][0];
                    d1[3] = ob[2 * pj + 1][1];
                }
                ptx::mma_bf16(d0, pa0, pa1, pa2, pa3, r[0], r[1]);
                ptx::mma_bf16(d1, pa0, pa1, pa2, pa3, r[2], r[3]);
                if constexpr (G16) {  // the lo parts of all 16 rows: a second product
                    ptx::mma_bf16(d0, la0, la1, la2, la3, r[0], r[1]);
                    ptx::mma_bf16(d1, la0, la1, la2, la3, r[2], r[3]);
                    o[2 * pj][0] = d0[0];
                    o[2 * pj][1] = d0[1];
                    o[2 * pj + 1][0] = d1[0];
                    o[2 * pj + 1][1] = d1[1];
                } else {              // rows g + 8 hold P_lo V: fold them into rows g
                    o[2 * pj][0] = d0[0] + d0[2];
                    o[2 * pj][1] = d0[1] + d0[3];
                    o[2 * pj + 1][0] = d1[0] + d1[2];
                    o[2 * pj + 1][1] = d1[1] + d1[3];
                }
                if constexpr (G16) {
                    ob[2 * pj][0] = d0[2];
                    ob[2 * pj][1] = d0[3];
                    ob[2 * pj + 1][0] = d1[2];
                    ob[2 * pj + 1][1] = d1[3];
                }
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
                const int64_t slot = ((int64_t)mt.b * a.S + mt.c) * a.wph + jw;
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

// ---------------------------------------------------------------------------
// INT8 consumer helpers
// ---------------------------------------------------------------------------
constexpr uint32_t kFlip = 0x80808080u;   // flips each byte's sign bit: byte = code + 128
constexpr uint32_t kBias = 0x64646464u;   // fp16 exponent byte of 1024
constexpr uint32_t kOnes = 0x3c003c00u;   // fp16x2 (1, 1)

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Two bytes of xf (= codes with the sign bit flipped), chosen by sel (0x4140:
// bytes 0,1; 0x4342: bytes 2,3), placed in the low mantissa bits of two fp16
// with exponent 2^10: the values 1024 + code + 128 exactly (10 mantissa bits).
__device__ __forceinline__ uint32_t biased_f16x2(uint32_t xf, uint32_t sel) {
    return prmt(xf, kBias, sel);
}

// The same pair with the bias removed: the exact codes as fp16x2.
__device__ __forceinline__ uint32_t codes_f16x2(uint32_t xf, uint32_t sel) {
    uint32_t r = biased_f16x2(xf, sel);
    asm("sub.rn.f16x2 %0, %0, %1;" : "+r"(r) : "r"(0x64806480u));  // 1152 = 1024 + 128
    return r;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

// Power of two 2^e (e clamped to [-126, 126], so 2^e and 2^-e are normal fp32
// values) with x * 2^e in [2^top, 2^(top + 1)) for a normal x > 0, from the
// exponent bits of x; a zero or subnormal x takes the clamp.
__device__ __forceinline__ float pow2_scale_for(float x, int top) {
    const int E = (int)((__float_as_uint(x) >> 23) & 0xffu) - 127;
    const int e = max(-126, min(126, top - E));
    return __uint_as_float((uint32_t)(e + 127) << 23);
}

// Query fragments of the INT8 consumer as int8 parts for the s8 MMA.
// Row g of the group is scaled by a power of two 2^e so that max|q| * 2^e lies
// in (L/2, L] with L = 8355711 = 127*65536 + 127*256 + 127, rounded to an
// integer q' (|q'| <= L) and split exactly into q' = 65536*hi + 256*mid + lo
// with hi in [-127, 127] and mid, lo in [-128, 127]; then
//   q'.k = 65536*(hi.k) + 256*(mid.k) + lo.k
// with the three dot products exact in int32.  The only approximation is the
// rounding q -> q' / 2^e: at most 1/(2 * 2^e) < max|q| / L (about 2^-23 of the
// row's largest element) per element, for rows whose largest element is at
// least 2^-104 (smaller rows take the scale 2^126).
// k-step kk (32 dims) of thread (g, tig) uses dims 16*tig + 4*kk + 0..3 (a0/a1)
// and 16*(tig + 4) + 4*kk + 0..3 (a2/a3), matching the K words it loads.
// Returns 1 / 2^e.
__device__ __forceinline__ float load_q_i8(const Args &a, int b, int row, bool live, int tig,
                                           uint32_t (&qh)[4][2], uint32_t (&qm)[4][2],
                                           uint32_t (&ql)[4][2]) {
    constexpr int D = 128;
    constexpr float kL = 8355711.f;
    float v[2][16];
    if (live) {
        const uint4 *qr = reinterpret_cast<const uint4 *>(a.q + ((int64_t)b * a.Hq + row) * D);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int c = tig + 4 * half;  // 16 dims = two uint4 of bf16
            const uint4 w0 = __ldg(qr + 2 * c), w1 = __ldg(qr + 2 * c + 1);
            const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                v[half][2 * i] = bf16_lo(w[i]);
                v[half][2 * i + 1] = bf16_hi(w[i]);
            }
        }
    } else {
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
            for (int i = 0; i < 16; ++i) v[half][i] = 0.f;
    }
    float mx = 0.f;
#pragma unroll
    for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fabsf(v[half][i]));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));  // the quad holds the whole row
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    // largest power of two sc with mx * sc <= L
    float sc = pow2_scale_for(mx, 22);
    if (mx * sc > kL) sc *= 0.5f;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            uint32_t hw = 0u, mw = 0u, lw = 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int qi = __float2int_rn(v[half][4 * w + e] * sc);
                const int r1 = (qi + 128) >> 8;   // qi = 256 * r1 + lo
                const int lo = qi - r1 * 256;
                const int hi = (r1 + 128) >> 8;   // r1 = 256 * hi + mid
                const int md = r1 - hi * 256;
                hw |= (uint32_t)(hi & 0xff) << (8 * e);
                mw |= (uint32_t)(md & 0xff) << (8 * e);
                lw |= (uint32_t)(lo & 0xff) << (8 * e);
            }
            qh[w][half] = hw;
            qm[w][half] = mw;
            ql[w][half] = lw;
        }
    }
    return 1.f / sc;   // exact: sc is a normal power of two
}

// Final write of one query row of the INT8 consumer: this thread holds dims
// 32*tig + nt (accumulator column 2*tig) and 32*tig + 16 + nt (2*tig + 1); the
// accumulators still carry the +1152 bias of V, removed here with lb = the
// same weights summed by the tensor core (sum_t p_t v-scale_t).
__device__ __forceinline__ void store_i8_row(const Args &a, const StageMeta &mt,
                                             const float (&oo)[16][2], float bias_sum,
                                             float lsum, float mm, int row, int tig, int jw) {
    constexpr int D = 128;
    const float corr = 1152.f * bias_sum;
    if (mt.flags & kDirect) {
        const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
        uint4 *dst = reinterpret_cast<uint4 *>(a.out + ((int64_t)mt.b * a.Hq + row) * D + 32 * tig);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                pk[i] = ptx::pack_bf16((oo[2 * i][c] - corr) * inv, (oo[2 * i + 1][c] - corr) * inv);
            dst[2 * c] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[2 * c + 1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
    } else {
        const int64_t slot = ((int64_t)mt.b * a.S + mt.c) * a.wph + jw;
        const int64_t r = slot * a.Hq + row;
        float4 *dst = reinterpret_cast<float4 *>(a.ws_acc + r * D + 32 * tig);
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                dst[4 * c + i] = make_float4(oo[4 * i][c] - corr, oo[4 * i + 1][c] - corr,
                                             oo[4 * i + 2][c] - corr, oo[4 * i + 3][c] - corr);
        if (tig == 0) *reinterpret_cast<float2 *>(a.ws_ml + r * 2) = make_float2(mm, lsum);
    }
}

// INT8 consumer (d = 128).  Same pipeline and softmax as the bf16 consumer; the
// tiles hold int8 codes, [head][token][128 bytes], 128-byte swizzled.
//  QK^T: int8 x int8 MMAs (m16n8k32) with exact int32 sums.  The dot product
//   over d is order-free, so thread (g, tig) takes, for k-step kk, the 32-bit
//   words kk of its two 16-byte chunks (dims 16*tig + 4*kk and 16*(tig+4) +
//   4*kk, 4 codes each) of its token row as its b0/b1 operands, and the query's
//   hi/mid/lo int8 parts (load_q_i8) use the same dims.  For G <= 8 one MMA takes
//   hi in rows g and mid in the otherwise empty rows g + 8, a second takes lo;
//   for G = 16 each part of rows g and g + 8 is one MMA.  Rows of odd g load their
//   two chunks in the other order (then swap), which keeps the shared-memory
//   reads conflict-free.
//  PV: n-tile nt, column g stands for dim 16*g + nt, so a thread reads 16 dims
//   (one 16-byte chunk) of each of its four token rows and byte-transposes
//   token pairs with prmt into (token, token+1) fp16 pairs, left biased by
//   +1152; one more MMA against an all-ones B sums the same fp16 weights, and
//   1152 times that sum is subtracted at the end.  Output column 2*tig (+1) of
//   n-tile nt is dim 32*tig + nt (+16).
//  The K scale multiplies the logit, the V scale the softmax weight.
//  A warp's two 16-token sub-tiles of a stage (one-byte pools: a stage carries
//  two per warp) take one softmax step together: both QK^T products, one max
//  over their 32 logits, one rescale of O, then both PV products.  That halves
//  the per-token softmax bookkeeping and gives the tensor and ALU pipes two
//  independent chains.

// Logits of rows g (and g + 8) of one 16-token sub-tile before the K scale:
// s0 holds tokens 2*tig, 2*tig + 1 (entries 0, 1: rows g; 2, 3: rows g + 8),
// s1 tokens 8 + 2*tig, 9 + 2*tig.
template <bool G16>
__device__ __forceinline__ void qk_i8(uint32_t kbase, int g, int tig, int odd,
                                      const uint32_t (&qh)[4][2], const uint32_t (&qm)[4][2],
                                      const uint32_t (&ql)[4][2],
                                      const uint32_t (&qhb)[G16 ? 4 : 1][2],
                                      const uint32_t (&qmb)[G16 ? 4 : 1][2],
                                      const uint32_t (&qlb)[G16 ? 4 : 1][2], float qs, float qsb,
                                      float (&s0)[4], float (&s1)[4]) {
    int sh[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}}, sl8[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
    int sm8[G16 ? 2 : 1][4] = {};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int t = 8 * nt + g;  // swizzle phase of row t is g
        const uint32_t rb = kbase + t * kBoxRow;
        const uint4 x0 = lds128(rb + (((tig + 4 * odd) ^ g) << 4));
        const uint4 x1 = lds128(rb + (((tig + 4 * (1 - odd)) ^ g) << 4));
        const uint4 lo = odd ? x1 : x0;  // dims 16*tig ..
        const uint4 hi = odd ? x0 : x1;  // dims 16*(tig+4) ..
        const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w}, wh[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            if constexpr (G16) {
                ptx::mma_s8(sh[nt], qh[kk][0], qhb[kk][0], qh[kk][1], qhb[kk][1], wl[kk], wh[kk]);
                ptx::mma_s8(sm8[nt], qm[kk][0], qmb[kk][0], qm[kk][1], qmb[kk][1], wl[kk],
                            wh[kk]);
                ptx::mma_s8(sl8[nt], ql[kk][0], qlb[kk][0], ql[kk][1], qlb[kk][1], wl[kk],
                            wh[kk]);
            } else {
                // G <= 8: the mid parts ride in the empty rows g + 8 of the hi MMA
                ptx::mma_s8(sh[nt], qh[kk][0], qm[kk][0], qh[kk][1], qm[kk][1], wl[kk], wh[kk]);
                ptx::mma_s8(sl8[nt], ql[kk][0], 0u, ql[kk][1], 0u, wl[kk], wh[kk]);
            }
        }
    }
    // q'.k = 65536 hi.k + 256 mid.k + lo.k: 256 hi.k + mid.k is exact in int32
    // (|hi.k| <= 128*127*127), the rest in fp32
    if constexpr (G16) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            s0[i] = fmaf((float)(sh[0][i] * 256 + sm8[0][i]), 256.f, (float)sl8[0][i]) *
                    (i < 2 ? qs : qsb);
            s1[i] = fmaf((float)(sh[1][i] * 256 + sm8[1][i]), 256.f, (float)sl8[1][i]) *
                    (i < 2 ? qs : qsb);
        }
    } else {  // hi . K in entries 0, 1, mid . K in entries 2, 3; lo . K in sl8 0, 1
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            s0[i] = fmaf((float)(sh[0][i] * 256 + sh[0][i + 2]), 256.f, (float)sl8[0][i]) * qs;
            s1[i] = fmaf((float)(sh[1][i] * 256 + sh[1][i + 2]), 256.f, (float)sl8[1][i]) * qs;
        }
        s0[2] = s0[3] = s1[2] = s1[3] = 0.f;
    }
}

// O += P (V + 1152) for one 16-token sub-tile; column g of n-tile nt is dim
// 16*g + nt.  (pa0, pa2): the fp16 weights (times the V scale) of rows g for
// tokens (2*tig, 2*tig + 1) and (8 + 2*tig, 9 + 2*tig); pa1, pa3 those of rows
// g + 8 (zero for G <= 8).  ol gathers the weights' sums (all-ones column).
template <bool G16>
__device__ __forceinline__ void pv_i8(uint32_t vbase, int g, int tig, uint32_t pa0, uint32_t pa1,
                                      uint32_t pa2, uint32_t pa3, float (&o)[16][2],
                                      float (&ob)[G16 ? 16 : 1][2], float (&ol)[4]) {
    const int t_a = 2 * tig, t_b = 8 + 2 * tig;
    const uint4 ra = lds128(vbase + t_a * kBoxRow + ((g ^ (t_a & 7)) << 4));
    const uint4 rb = lds128(vbase + (t_a + 1) * kBoxRow + ((g ^ ((t_a + 1) & 7)) << 4));
    const uint4 rc = lds128(vbase + t_b * kBoxRow + ((g ^ (t_b & 7)) << 4));
    const uint4 rd = lds128(vbase + (t_b + 1) * kBoxRow + ((g ^ ((t_b + 1) & 7)) << 4));
    const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w}, wb[4] = {rb.x, rb.y, rb.z, rb.w};
    const uint32_t wc[4] = {rc.x, rc.y, rc.z, rc.w}, wd[4] = {rd.x, rd.y, rd.z, rd.w};
    {
        float dd[4] = {ol[0], ol[1], ol[2], ol[3]};
        ptx::mma_f16(dd, pa0, pa1, pa2, pa3, kOnes, kOnes);
#pragma unroll
        for (int i = 0; i < 4; ++i) ol[i] = dd[i];
    }
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t fa = wa[w] ^ kFlip, fb = wb[w] ^ kFlip;
        const uint32_t fc = wc[w] ^ kFlip, fd = wd[w] ^ kFlip;
        const uint32_t X = prmt(fa, fb, 0x5140u), Y = prmt(fa, fb, 0x7362u);
        const uint32_t Z = prmt(fc, fd, 0x5140u), U = prmt(fc, fd, 0x7362u);
        const uint32_t b0[4] = {biased_f16x2(X, 0x4140u), biased_f16x2(X, 0x4342u),
                                biased_f16x2(Y, 0x4140u), biased_f16x2(Y, 0x4342u)};
        const uint32_t b1[4] = {biased_f16x2(Z, 0x4140u), biased_f16x2(Z, 0x4342u),
                                biased_f16x2(U, 0x4140u), biased_f16x2(U, 0x4342u)};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int nt = 4 * w + i;
            float dd[4] = {o[nt][0], o[nt][1], 0.f, 0.f};
            if constexpr (G16) {
                dd[2] = ob[nt][0];
                dd[3] = ob[nt][1];
            }
            ptx::mma_f16(dd, pa0, pa1, pa2, pa3, b0[i], b1[i]);
            o[nt][0] = dd[0];
            o[nt][1] = dd[1];
            if constexpr (G16) {
                ob[nt][0] = dd[2];
                ob[nt][1] = dd[3];
            }
        }
    }
}

// One online-softmax step of one query row over the 8 logits a thread holds for
// a sub-tile pair (x[0..3]: sub-tile A, x[4..7]: B; -inf where masked) with the
// quad's other 24: updates (m, l), returns alpha = 2^(m_old - m_new) and the
// weights p (2^(x - m_new)).
__device__ __forceinline__ float softmax_pair_step(const float (&x)[8], float &m, float &l,
                                                   float (&p)[8]) {
    float mx = fmaxf(fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3])),
                     fmaxf(fmaxf(x[4], x[5]), fmaxf(x[6], x[7])));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    const float mn = fmaxf(m, mx);
    const float mu = mn == -INFINITY ? 0.f : mn;
    const float alpha = ex2_fast(m - mu);
#pragma unroll
    for (int i = 0; i < 8; ++i) p[i] = ex2_fast(x[i] - mu);
    l = l * alpha + (((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7])));
    m = mn;
    return alpha;
}

template <bool G16>
__device__ __forceinline__ void consumer_i8(const Args &a, uint8_t *stages, StageMeta *meta,
                                            uint64_t *full, uint64_t *empty) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = warp % a.Hkv, jw = warp / a.Hkv;
    const int g = lane >> 2, tig = lane & 3;
    const int odd = g & 1;
    const uint32_t stage0 = ptx::smem_u32(stages);
    const uint32_t head_off = (uint32_t)(h * kTile * kBoxRow);
    const uint32_t sub_bytes = (uint32_t)a.box_bytes;           // one box per sub-tile (d = 128)
    const uint32_t sc_sub = (uint32_t)(kTile * a.Hkv * 4);      // scale rows of one sub-tile
    const int hs = a.Hkv * 4;                                   // bytes between token scale rows
    const int t_a = 2 * tig, t_b = 8 + 2 * tig;                 // this thread's token pairs

    uint32_t qh[4][2], qm[4][2], ql[4][2];                // rows g: hi / mid / lo parts
    uint32_t qhb[G16 ? 4 : 1][2], qmb[G16 ? 4 : 1][2], qlb[G16 ? 4 : 1][2];  // rows g + 8
    float qs = 0.f, qsb = 0.f;                            // 1 / 2^e of rows g and g + 8
    float o[16][2];
    float ob[G16 ? 16 : 1][2];
    float ol[4];  // sums of the fp16 weights (all-ones column), rows g and g + 8
    float m = -INFINITY, l = 0.f, mb = -INFINITY, lb = 0.f;
    int q_b = first_unit_seq(a);   // the sequence whose query the registers hold
    if (q_b >= 0) {
        qs = load_q_i8(a, q_b, h * a.G + g, g < a.G, tig, qh, qm, ql);
        if constexpr (G16)
            qsb = load_q_i8(a, q_b, h * a.G + g + 8, g + 8 < a.G, tig, qhb, qmb, qlb);
    }
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
            if (mt.b != q_b) {
                qs = load_q_i8(a, mt.b, h * a.G + g, g < a.G, tig, qh, qm, ql);
                if constexpr (G16)
                    qsb = load_q_i8(a, mt.b, h * a.G + g + 8, g + 8 < a.G, tig, qhb, qmb, qlb);
            }
            q_b = -1;
            m = -INFINITY;
            l = 0.f;
            mb = -INFINITY;
            lb = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) ol[i] = 0.f;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                o[nt][0] = o[nt][1] = 0.f;
                if constexpr (G16) ob[nt][0] = ob[nt][1] = 0.f;
            }
        }
        // this warp's two sub-tiles of the stage (A before B in token order)
        const int jA = jw, jB = jw + a.wph;
        const int nvA = max(0, min(kTile, mt.te - (mt.ts + kTile * jA)));
        const int nvB = max(0, min(kTile, mt.te - (mt.ts + kTile * jB)));
        const bool liveA = nvA > 0 && !((mt.bad >> jA) & 1);
        const bool liveB = nvB > 0 && !((mt.bad >> jB) & 1);
        if (liveA || liveB) {
            // ---- S = Q K^T on int8 tensor cores: K codes straight from shared memory
            float sA0[4] = {0.f, 0.f, 0.f, 0.f}, sA1[4] = {0.f, 0.f, 0.f, 0.f};
            float sB0[4] = {0.f, 0.f, 0.f, 0.f}, sB1[4] = {0.f, 0.f, 0.f, 0.f};
            if (liveA)
                qk_i8<G16>(sb + jA * sub_bytes + head_off, g, tig, odd, qh, qm, ql, qhb, qmb,
                           qlb, qs, qsb, sA0, sA1);
            if (liveB)
                qk_i8<G16>(sb + jB * sub_bytes + head_off, g, tig, odd, qh, qm, ql, qhb, qmb,
                           qlb, qs, qsb, sB0, sB1);
            // ---- online softmax over both sub-tiles; K scale folded into the logit
            const bool va[8] = {liveA && t_a < nvA, liveA && t_a + 1 < nvA,
                                liveA && t_b < nvA, liveA && t_b + 1 < nvA,
                                liveB && t_a < nvB, liveB && t_a + 1 < nvB,
                                liveB && t_b < nvB, liveB && t_b + 1 < nvB};
            const int tok[4] = {t_a, t_a + 1, t_b, t_b + 1};
            const uint32_t ksA = sb + a.ks_off + jA * sc_sub + h * 4;
            const uint32_t ksB = sb + a.ks_off + jB * sc_sub + h * 4;
            const uint32_t vsA = sb + a.vs_off + jA * sc_sub + h * 4;
            const uint32_t vsB = sb + a.vs_off + jB * sc_sub + h * 4;
            const float sl = a.scale_log2;
            float kf[8], vf[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                kf[i] = va[i] ? lds_f32(ksA + tok[i] * hs) * sl : 0.f;
                kf[4 + i] = va[4 + i] ? lds_f32(ksB + tok[i] * hs) * sl : 0.f;
                vf[i] = va[i] ? lds_f32(vsA + tok[i] * hs) : 0.f;
                vf[4 + i] = va[4 + i] ? lds_f32(vsB + tok[i] * hs) : 0.f;
            }
            const float rawg[8] = {sA0[0], sA0[1], sA1[0], sA1[1], sB0[0], sB0[1], sB1[0], sB1[1]};
            float x[8], p[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = va[i] ? rawg[i] * kf[i] : -INFINITY;
            const float alpha = softmax_pair_step(x, m, l, p);
            const uint32_t pA0 = ptx::pack_f16(p[0] * vf[0], p[1] * vf[1]);
            const uint32_t pA2 = ptx::pack_f16(p[2] * vf[2], p[3] * vf[3]);
            const uint32_t pB0 = ptx::pack_f16(p[4] * vf[4], p[5] * vf[5]);
            const uint32_t pB2 = ptx::pack_f16(p[6] * vf[6], p[7] * vf[7]);
            uint32_t pA1 = 0u, pA3 = 0u, pB1 = 0u, pB3 = 0u;
            float alphab = 1.f;
            if constexpr (G16) {
                const float rawb[8] = {sA0[2], sA0[3], sA1[2], sA1[3],
                                       sB0[2], sB0[3], sB1[2], sB1[3]};
                float y[8], q[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) y[i] = va[i] ? rawb[i] * kf[i] : -INFINITY;
                alphab = softmax_pair_step(y, mb, lb, q);
                pA1 = ptx::pack_f16(q[0] * vf[0], q[1] * vf[1]);
                pA3 = ptx::pack_f16(q[2] * vf[2], q[3] * vf[3]);
                pB1 = ptx::pack_f16(q[4] * vf[4], q[5] * vf[5]);
                pB3 = ptx::pack_f16(q[6] * vf[6], q[7] * vf[7]);
            }
            // rescale only when some row maximum moved (alpha == 1 exactly otherwise)
            if (__any_sync(kFull, alpha != 1.f || alphab != 1.f)) {
                ol[0] *= alpha;
                ol[1] *= alpha;
                ol[2] *= alphab;
                ol[3] *= alphab;
#pragma unroll
                for (int nt = 0; nt < 16; ++nt) {
                    o[nt][0] *= alpha;
                    o[nt][1] *= alpha;
                    if constexpr (G16) {
                        ob[nt][0] *= alphab;
                        ob[nt][1] *= alphab;
                    }
                }
            }
            // ---- O += P (V + 1152), sub-tile A then B
            if (liveA)
                pv_i8<G16>(sb + a.v_off + jA * sub_bytes + head_off, g, tig, pA0, pA1, pA2, pA3,
                           o, ob, ol);
            if (liveB)
                pv_i8<G16>(sb + a.v_off + jB * sub_bytes + head_off, g, tig, pB0, pB1, pB2, pB3,
                           o, ob, ol);
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
            if (g < a.G) store_i8_row(a, mt, o, ol[0], lt, m, row, tig, jw);
            if constexpr (G16) {
                if (g + 8 < a.G) store_i8_row(a, mt, ob, ol[2], ltb, mb, row + 8, tig, jw);
            }
        }
        if (++stage == a.nstage) {
            stage = 0;
            phase ^= 1u;
        }
    }
}

// Two e4m3 codes (one 16-bit half of w; low byte first) -> exact fp16x2.
__device__ __forceinline__ void e4m3_word_to_f16x2(uint32_t w, uint32_t &lo, uint32_t &hi) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// Query fragments (fp16) for the FP8 consumer: k-step kk (16 dims) of thread
// (g, tig) uses dims 16*(tig + 4*(kk/4)) + 4*(kk%4) + 0..3, the dims of the K
// word it converts (see consumer_fp8).  The row is first scaled by a power of
// two 2^e that puts its largest magnitude in [2^14, 2^15): every bf16 query
// then fits fp16 without overflow (|q| above 65504 included), and every element
// no smaller than 2^-32 of the row's largest converts exactly (fp16 keeps 11
// significant bits against bf16's 8); smaller ones round with an error below
// 2^-39 of the largest.  Returns 1 / 2^e, which the logit takes back.
__device__ __forceinline__ float load_q_f16perm(const Args &a, int b, int row, bool live, int tig,
                                                uint32_t (&qa)[8][2]) {
    constexpr int D = 128;
    const uint4 *qr = reinterpret_cast<const uint4 *>(a.q + ((int64_t)b * a.Hq + row) * D);
    uint4 w[4];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int c = tig + 4 * half;  // 16 dims = two uint4 of bf16
        w[2 * half] = live ? __ldg(qr + 2 * c) : make_uint4(0u, 0u, 0u, 0u);
        w[2 * half + 1] = live ? __ldg(qr + 2 * c + 1) : make_uint4(0u, 0u, 0u, 0u);
    }
    // |bf16| of a pair word is the word with both sign bits cleared; compare the
    // halves as floats
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t u[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            mx = fmaxf(mx, fmaxf(fabsf(bf16_lo(u[j])), fabsf(bf16_hi(u[j]))));
    }
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));  // the quad holds the whole row
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    const float sc = pow2_scale_for(mx, 14);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        uint32_t f[8];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const uint4 v = w[2 * half + k];
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
                f[4 * k + i] = ptx::pack_f16(bf16_lo(u[i]) * sc, bf16_hi(u[i]) * sc);
        }
#pragma unroll
        for (int kw = 0; kw < 4; ++kw) {
            qa[4 * half + kw][0] = f[2 * kw];
            qa[4 * half + kw][1] = f[2 * kw + 1];
        }
    }
    return 1.f / sc;   // exact: sc is a normal power of two
}

// FP8 (e4m3) consumer (d = 128).  Same pipeline and softmax as the bf16
// consumer; tiles hold e4m3 codes, [head][token][128 bytes], 128-byte swizzled,
// converted exactly to fp16 in registers (every e4m3 value is an fp16).
//  QK^T: k-step kk of thread (g, tig) converts word kk of its two 16-byte
//   chunks (dims 16*(tig + 4*(kk/4)) + 4*(kk%4) + 0..3) into its b0/b1 pair;
//   the query fragments use the same dims (load_q_f16perm).
//  PV: as in the INT8 consumer -- n-tile nt, column g is dim 16*g + nt; token
//   pairs are byte-transposed with prmt before the conversion.
//  As in the INT8 consumer, a warp's two sub-tiles of a stage take one softmax
//  step together.

// Logits of rows g (and g + 8) of one 16-token sub-tile, before scale and the
// query's 2^-e (layout as qk_i8).
template <bool G16>
__device__ __forceinline__ void qk_fp8(uint32_t kbase, int g, int tig, int odd,
                                       const uint32_t (&qa)[8][2],
                                       const uint32_t (&qb)[G16 ? 8 : 1][2], float (&s0)[4],
                                       float (&s1)[4]) {
    float e0[4] = {0.f, 0.f, 0.f, 0.f}, e1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) s0[i] = s1[i] = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int t = 8 * nt + g;  // swizzle phase of row t is g
        const uint32_t rb = kbase + t * kBoxRow;
        const uint4 x0 = lds128(rb + (((tig + 4 * odd) ^ g) << 4));
        const uint4 x1 = lds128(rb + (((tig + 4 * (1 - odd)) ^ g) << 4));
        const uint4 lo = odd ? x1 : x0;  // dims 16*tig ..
        const uint4 hi = odd ? x0 : x1;  // dims 16*(tig+4) ..
        const uint32_t wd[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t b0, b1;
            e4m3_word_to_f16x2(wd[kk], b0, b1);
            // even and odd k-steps in separate accumulators: two independent chains
            float(&acc)[4] = nt == 0 ? ((kk & 1) ? e0 : s0) : ((kk & 1) ? e1 : s1);
            if constexpr (G16)
                ptx::mma_f16(acc, qa[kk][0], qb[kk][0], qa[kk][1], qb[kk][1], b0, b1);
            else
                ptx::mma_f16(acc, qa[kk][0], 0u, qa[kk][1], 0u, b0, b1);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        s0[i] += e0[i];
        s1[i] += e1[i];
    }
}

// O += P V for one 16-token sub-tile of e4m3 codes (column g of n-tile nt is dim
// 16*g + nt).  Masked tokens have P = 0; their codes may be NaN (0x7f), so the
// rows of tokens outside [0, nv) are zeroed.
template <bool G16>
__device__ __forceinline__ void pv_fp8(uint32_t vbase, int g, int tig, int nv, uint32_t pa0,
                                       uint32_t pa1, uint32_t pa2, uint32_t pa3,
                                       float (&o)[16][2], float (&ob)[G16 ? 16 : 1][2]) {
    const int t_a = 2 * tig, t_b = 8 + 2 * tig;
    const uint4 ra = lds128(vbase + t_a * kBoxRow + ((g ^ (t_a & 7)) << 4));
    const uint4 rb = lds128(vbase + (t_a + 1) * kBoxRow + ((g ^ ((t_a + 1) & 7)) << 4));
    const uint4 rc = lds128(vbase + t_b * kBoxRow + ((g ^ (t_b & 7)) << 4));
    const uint4 rd = lds128(vbase + (t_b + 1) * kBoxRow + ((g ^ ((t_b + 1) & 7)) << 4));
    const uint32_t za = t_a < nv ? ~0u : 0u, zb = t_a + 1 < nv ? ~0u : 0u;
    const uint32_t zc = t_b < nv ? ~0u : 0u, zd = t_b + 1 < nv ? ~0u : 0u;
    const uint32_t wa[4] = {ra.x & za, ra.y & za, ra.z & za, ra.w & za};
    const uint32_t wb[4] = {rb.x & zb, rb.y & zb, rb.z & zb, rb.w & zb};
    const uint32_t wc[4] = {rc.x & zc, rc.y & zc, rc.z & zc, rc.w & zc};
    const uint32_t wdv[4] = {rd.x & zd, rd.y & zd, rd.z & zd, rd.w & zd};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t X = prmt(wa[w], wb[w], 0x5140u), Y = prmt(wa[w], wb[w], 0x7362u);
        const uint32_t Z = prmt(wc[w], wdv[w], 0x5140u), U = prmt(wc[w], wdv[w], 0x7362u);
        uint32_t b0[4], b1[4];
        e4m3_word_to_f16x2(X, b0[0], b0[1]);
        e4m3_word_to_f16x2(Y, b0[2], b0[3]);
        e4m3_word_to_f16x2(Z, b1[0], b1[1]);
        e4m3_word_to_f16x2(U, b1[2], b1[3]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int nt = 4 * w + i;
            float dd[4] = {o[nt][0], o[nt][1], 0.f, 0.f};
            if constexpr (G16) {
                dd[2] = ob[nt][0];
                dd[3] = ob[nt][1];
            }
            ptx::mma_f16(dd, pa0, pa1, pa2, pa3, b0[i], b1[i]);
            o[nt][0] = dd[0];
            o[nt][1] = dd[1];
            if constexpr (G16) {
                ob[nt][0] = dd[2];
                ob[nt][1] = dd[3];
            }
        }
    }
}

template <bool G16>
__device__ __forceinline__ void consumer_fp8(const Args &a, uint8_t *stages, StageMeta *meta,
                                             uint64_t *full, uint64_t *empty) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = warp % a.Hkv, jw = warp / a.Hkv;
    const int g = lane >> 2, tig = lane & 3;
    const int odd = g & 1;
    const uint32_t stage0 = ptx::smem_u32(stages);
    const uint32_t head_off = (uint32_t)(h * kTile * kBoxRow);
    const uint32_t sub_bytes = (uint32_t)a.box_bytes;
    const int t_a = 2 * tig, t_b = 8 + 2 * tig;   // this thread's token pairs

    uint32_t qa[8][2];
    uint32_t qb[G16 ? 8 : 1][2];
    float qs = 1.f, qsb = 1.f;  // 1 / 2^e of rows g and g + 8 (load_q_f16perm)
    float o[16][2];
    float ob[G16 ? 16 : 1][2];
    float m = -INFINITY, l = 0.f, mb = -INFINITY, lb = 0.f;
    // (no early load of the first unit's query here: it measured slower on this
    // consumer, 199.6 -> 201.2 us per call on the c5 shape, where INT8 gained 2 %)
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
            qs = load_q_f16perm(a, mt.b, h * a.G + g, g < a.G, tig, qa);
            if constexpr (G16) {
                uint32_t t[8][2];
                qsb = load_q_f16perm(a, mt.b, h * a.G + g + 8, g + 8 < a.G, tig, t);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    qb[kk][0] = t[kk][0];
                    qb[kk][1] = t[kk][1];
                }
            }
            m = -INFINITY;
            l = 0.f;
            mb = -INFINITY;
            lb = 0.f;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                o[nt][0] = o[nt][1] = 0.f;
                if constexpr (G16) ob[nt][0] = ob[nt][1] = 0.f;
            }
        }
        // this warp's two sub-tiles of the stage (A before B in token order)
        const int jA = jw, jB = jw + a.wph;
        const int nvA0 = max(0, min(kTile, mt.te - (mt.ts + kTile * jA)));
        const int nvB0 = max(0, min(kTile, mt.te - (mt.ts + kTile * jB)));
        const bool liveA = nvA0 > 0 && !((mt.bad >> jA) & 1);
        const bool liveB = nvB0 > 0 && !((mt.bad >> jB) & 1);
        if (liveA || liveB) {
            const int nvA = liveA ? nvA0 : 0, nvB = liveB ? nvB0 : 0;
            // ---- S = Q K^T (exact fp16 values of the codes)
            float sA0[4] = {0.f, 0.f, 0.f, 0.f}, sA1[4] = {0.f, 0.f, 0.f, 0.f};
            float sB0[4] = {0.f, 0.f, 0.f, 0.f}, sB1[4] = {0.f, 0.f, 0.f, 0.f};
            if (liveA) qk_fp8<G16>(sb + jA * sub_bytes + head_off, g, tig, odd, qa, qb, sA0, sA1);
            if (liveB) qk_fp8<G16>(sb + jB * sub_bytes + head_off, g, tig, odd, qa, qb, sB0, sB1);
            // ---- online softmax over both sub-tiles (the query's 2^-e folded in, exact)
            const bool va[8] = {t_a < nvA, t_a + 1 < nvA, t_b < nvA, t_b + 1 < nvA,
                                t_a < nvB, t_a + 1 < nvB, t_b < nvB, t_b + 1 < nvB};
            const float sl = a.scale_log2 * qs;
            const float rawg[8] = {sA0[0], sA0[1], sA1[0], sA1[1], sB0[0], sB0[1], sB1[0], sB1[1]};
            float x[8], p[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = va[i] ? rawg[i] * sl : -INFINITY;
            const float alpha = softmax_pair_step(x, m, l, p);
            const uint32_t pA0 = ptx::pack_f16(p[0], p[1]), pA2 = ptx::pack_f16(p[2], p[3]);
            const uint32_t pB0 = ptx::pack_f16(p[4], p[5]), pB2 = ptx::pack_f16(p[6], p[7]);
            uint32_t pA1 = 0u, pA3 = 0u, pB1 = 0u, pB3 = 0u;
            float alphab = 1.f;
            if constexpr (G16) {
                const float slb = a.scale_log2 * qsb;
                const float rawb[8] = {sA0[2], sA0[3], sA1[2], sA1[3],
                                       sB0[2], sB0[3], sB1[2], sB1[3]};
                float y[8], q[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) y[i] = va[i] ? rawb[i] * slb : -INFINITY;
                alphab = softmax_pair_step(y, mb, lb, q);
                pA1 = ptx::pack_f16(q[0], q[1]);
                pA3 = ptx::pack_f16(q[2], q[3]);
                pB1 = ptx::pack_f16(q[4], q[5]);
                pB3 = ptx::pack_f16(q[6], q[7]);
            }
            if (__any_sync(kFull, alpha != 1.f || alphab != 1.f)) {
#pragma unroll
                for (int nt = 0; nt < 16; ++nt) {
                    o[nt][0] *= alpha;
                    o[nt][1] *= alpha;
                    if constexpr (G16) {
                        ob[nt][0] *= alphab;
                        ob[nt][1] *= alphab;
                    }
                }
            }
            // ---- O += P V, sub-tile A then B
            if (liveA)
                pv_fp8<G16>(sb + a.v_off + jA * sub_bytes + head_off, g, tig, nvA, pA0, pA1, pA2,
                            pA3, o, ob);
            if (liveB)
                pv_fp8<G16>(sb + a.v_off + jB * sub_bytes + head_off, g, tig, nvB, pB0, pB1, pB2,
                            pB3, o, ob);
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
            if (g < a.G) store_i8_row(a, mt, o, 0.f, lt, m, row, tig, jw);
            if constexpr (G16) {
                if (g + 8 < a.G) store_i8_row(a, mt, ob, 0.f, ltb, mb, row + 8, tig, jw);
            }
        }
        if (++stage == a.nstage) {
            stage = 0;
            phase ^= 1u;
        }
    }
}

template <int D, bool G16, int KV>
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
    if (threadIdx.x == kConsumerWarps * 32) {   // the tensor maps are launch parameters
        ptx::prefetch_tensormap(&kmap);
        ptx::prefetch_tensormap(&vmap);
    }
    __syncthreads();
    // launched programmatically after the plan kernel: the set-up above overlaps
    // it; the plan (and, through it, the KV append before it) is complete here.
    // The merge launch is released only after this wait, so the selection CTAs at
    // its front may read the score pool the append wrote without waiting themselves.
    ptx::grid_dependency_wait();
    ptx::grid_launch_dependents();
    if ((threadIdx.x >> 5) == kConsumerWarps)
        producer<D, KV>(&kmap, &vmap, a, stages, meta, full, empty);
    else if constexpr (KV == kKvInt8)
        consumer_i8<G16>(a, stages, meta, full, empty);
    else if constexpr (KV == kKvFp8)
        consumer_fp8<G16>(a, stages, meta, full, empty);
    else
        consumer<D, G16>(a, stages, meta, full, empty);
}

// Merge of the partials of one (sequence, query head) in slot order:
// M = max_s m_s, out = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s.
// One thread per dim walks the partials; for sequences cut into many partitions
// (long contexts) the D/32 warps of the CTA split the partials instead (lane:
// D/32 dims, float4 / float2 loads) and add their sums in warp order, so the
// loads of many partials are in flight at once.
constexpr int kWideMerge = 32;   // partials per row from which the warps split them

template <int D>
__device__ __forceinline__ void merge_wide(const Args &a, int64_t bh, int i, int cnt,
                                           int64_t base) {
    constexpr int W = D / 32, E = D / 32;
    __shared__ float s_max[W], s_l[W];
    __shared__ float s_acc[W][D];
    const int e = threadIdx.x, warp = e >> 5, lane = e & 31;
    float M = -INFINITY;
    for (int s = e; s < cnt; s += D) M = fmaxf(M, a.ws_ml[((base + s) * a.Hq + i) * 2]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
    if (lane == 0) s_max[warp] = M;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, s_max[w]);
    float L = 0.f, A[E];
#pragma unroll
    for (int k = 0; k < E; ++k) A[k] = 0.f;
    if (M != -INFINITY) {
#pragma unroll 8
        for (int s = warp; s < cnt; s += W) {
            const int64_t r = (base + s) * a.Hq + i;
            const float2 ml = *reinterpret_cast<const float2 *>(a.ws_ml + r * 2);
            const float f = exp2f(ml.x - M);
            L = fmaf(ml.y, f, L);
            const float *src = a.ws_acc + r * D + lane * E;
            if constexpr (E == 4) {
                const float4 v = *reinterpret_cast<const float4 *>(src);
                A[0] = fmaf(v.x, f, A[0]);
                A[1] = fmaf(v.y, f, A[1]);
                A[2] = fmaf(v.z, f, A[2]);
                A[3] = fmaf(v.w, f, A[3]);
            } else {
                const float2 v = *reinterpret_cast<const float2 *>(src);
                A[0] = fmaf(v.x, f, A[0]);
                A[1] = fmaf(v.y, f, A[1]);
            }
        }
    }
#pragma unroll
    for (int k = 0; k < E; ++k) s_acc[warp][lane * E + k] = A[k];
    if (lane == 0) s_l[warp] = L;
    __syncthreads();
    float As = 0.f, Ls = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) {
        As += s_acc[w][e];
        Ls += s_l[w];
    }
    a.out[bh * D + e] = f32_to_bf16_rn(Ls > 0.f ? As / Ls : 0.f);
}

template <int D>
__global__ void __launch_bounds__(D) merge_tc_kernel(const Args a) {
    // the next kernel may start its set-up now; its own wait still covers this one
    ptx::grid_launch_dependents();
    ptx::grid_dependency_wait();  // the decode kernel's partials are complete
    if (a.hdr->sig != a.sig) return;  // no plan for these sizes (flagged by the decode)
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / a.Hq), i = (int)(bh % a.Hq);
    const int e = threadIdx.x;
    const int nsb = a.ns[b];
    if (nsb == 1 && a.wph == 1) return;  // written directly by the decode kernel
    const int cnt = nsb * a.wph;
    const int64_t base = (int64_t)b * a.S * a.wph;
    if (cnt > kWideMerge) {   // uniform over the CTA
        merge_wide<D>(a, bh, i, cnt, base);
        return;
    }
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

// Merge with one warp per output row (b, i), 8 rows per CTA: lane j takes the
// (m, l) of partial c0 + j of each 32-partial chunk, the row maximum and the
// weights f = 2^(m - M) come from warp shuffles, and each lane accumulates its
// D/32 dims of sum_s f_s acc_s in slot order.  Used when every row has few
// partials (short contexts), where one small CTA per row spends most of its time
// starting and waiting.  The plan's signature, the piece count, the first 32
// (m, l) pairs and the first kAhead partials' accumulators do not depend on one
// another: they are loaded in one round (slots past the sequence's count are read
// but never used; every slot of the sequence's S * wph exists), so a row with at
// most kAhead partials waits for one round trip instead of four.
constexpr int kRowsPerMergeCta = 8;
constexpr int kAhead = 8;

static_assert(32 * kRowsPerMergeCta == kSelThreads, "selection CTAs share the merge's block");

template <int D>
__global__ void __launch_bounds__(32 * kRowsPerMergeCta) merge_rows_kernel(const Args a) {
    constexpr int E = D / 32;
    // the next kernel may start its set-up now; its own wait still covers this one
    ptx::grid_launch_dependents();
    if ((int)blockIdx.x < a.sel_ctas) {
        // the block selection of sequence blockIdx.x: it reads the score pool and the
        // tables only, written before the decode kernel's dependency wait released
        // this launch, so it runs beside the decode kernel
        select_pooled_cta(a.sel_evict, a.sel_means, a.sel_scores, a.bt, a.ctx_lens, a.err, a.MB,
                          a.Hkv, a.bs, a.N, (int)blockIdx.x);
        return;
    }
    ptx::grid_dependency_wait();  // the decode kernel's partials are complete
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t bh = (int64_t)(blockIdx.x - a.sel_ctas) * kRowsPerMergeCta + warp;
    if (bh >= (int64_t)a.B * a.Hq) return;
    const int b = (int)(bh / a.Hq), i = (int)(bh % a.Hq);
    const int cap = a.S * a.wph;               // partial slots of one sequence
    const int64_t base = (int64_t)b * cap;
    const unsigned long long hsig = a.hdr->sig;
    const int nsb = a.ns[b];
    float2 ml0 = make_float2(-INFINITY, 0.f);
    if (lane < cap) ml0 = *reinterpret_cast<const float2 *>(a.ws_ml + ((base + lane) * a.Hq + i) * 2);
    float va[kAhead][E];
#pragma unroll
    for (int j = 0; j < kAhead; ++j) {
        if (j < cap) {
            const float *src = a.ws_acc + ((base + j) * a.Hq + i) * D + lane * E;
            if constexpr (E == 4) {
                const float4 v = *reinterpret_cast<const float4 *>(src);
                va[j][0] = v.x, va[j][1] = v.y, va[j][2] = v.z, va[j][3] = v.w;
            } else {
                const float2 v = *reinterpret_cast<const float2 *>(src);
                va[j][0] = v.x, va[j][1] = v.y;
            }
        }
    }
    if (hsig != a.sig) return;  // no plan for these sizes (flagged by the decode)
    if (nsb == 1 && a.wph == 1) return;  // written directly by the decode kernel
    const int cnt = nsb * a.wph;
    float M = lane < cnt ? ml0.x : -INFINITY;
    for (int s = lane + 32; s < cnt; s += 32) M = fmaxf(M, a.ws_ml[((base + s) * a.Hq + i) * 2]);
    M = warp_max(M);
    float L = 0.f, A[E];
#pragma unroll
    for (int k = 0; k < E; ++k) A[k] = 0.f;
    if (M != -INFINITY) {
        for (int c0 = 0; c0 < cnt; c0 += 32) {
            float f = 0.f;
            if (c0 + lane < cnt) {
                const float2 ml = c0 == 0 ? ml0
                                          : *reinterpret_cast<const float2 *>(
                                                a.ws_ml + ((base + c0 + lane) * a.Hq + i) * 2);
                f = exp2f(ml.x - M);
                L = fmaf(ml.y, f, L);
            }
            const int n = min(32, cnt - c0);
            int j = 0;
            if (c0 == 0) {   // the partials loaded ahead
#pragma unroll
                for (int k = 0; k < kAhead; ++k) {
                    if (k < n) {
                        const float fj = __shfl_sync(kFull, f, k);
#pragma unroll
                        for (int e = 0; e < E; ++e) A[e] = fmaf(va[k][e], fj, A[e]);
                    }
                }
                j = kAhead;
            }
#pragma unroll 8
            for (; j < n; ++j) {
                const float fj = __shfl_sync(kFull, f, j);
                const float *src = a.ws_acc + ((base + c0 + j) * a.Hq + i) * D + lane * E;
                if constexpr (E == 4) {
                    const float4 v = *reinterpret_cast<const float4 *>(src);
                    A[0] = fmaf(v.x, fj, A[0]);
                    A[1] = fmaf(v.y, fj, A[1]);
                    A[2] = fmaf(v.z, fj, A[2]);
                    A[3] = fmaf(v.w, fj, A[3]);
                } else {
                    const float2 v = *reinterpret_cast<const float2 *>(src);
                    A[0] = fmaf(v.x, fj, A[0]);
                    A[1] = fmaf(v.y, fj, A[1]);
                }
            }
        }
        L = warp_sum(L);
    }
    uint16_t *o = a.out + bh * D + lane * E;
#pragma unroll
    for (int k = 0; k < E; ++k) o[k] = f32_to_bf16_rn(L > 0.f ? A[k] / L : 0.f);
}

// ---------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------
// Launch with programmatic stream serialization: the kernel may start while the
// previous kernel in the stream is still running; it calls griddepcontrol.wait
// before it touches anything the previous kernel produced.
template <typename... KArgs, typename... Args2>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args2 &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args2>(args)...);
}

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

// Element width (bytes) the tensor maps use to move pool rows.  A TMA copy
// does not interpret the data, so bf16 and int8 pools are both moved as this
// many-byte elements; the box is 128 bytes of d either way.
constexpr int kTmaElt = 2;

// The pool is viewed as 5-D (innermost first):
//   128 bytes of one (token, head) vector | slot in block | kv head |
//   128-byte slice of the vector | physical block,
// and one TMA box is (128 bytes, 16 tokens, Hkv heads, 1, 1): in shared memory
// [head][token][128 bytes], 128-byte swizzled, so each head's 16 token rows are
// 16 consecutive swizzled rows that ldmatrix / 16-byte loads read without bank
// conflicts.
bool encode_pool_map(CUtensorMap *map, const void *base, int64_t N, int bs, int Hkv, int d,
                     int64_t block_stride, bool int8) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int64_t row = (int64_t)d * (int8 ? 1 : 2);  // bytes of one (token, head) vector
    const int inner = 128 / kTmaElt;                    // elements in one 128-byte box row
    const cuuint64_t dims[5] = {(cuuint64_t)inner, (cuuint64_t)bs, (cuuint64_t)Hkv,
                                (cuuint64_t)(row / 128), (cuuint64_t)N};
    const cuuint64_t strides[4] = {(cuuint64_t)(Hkv * row), (cuuint64_t)row, 128,
                                   (cuuint64_t)(block_stride * (int8 ? 1 : 2))};
    const cuuint32_t box[5] = {(cuuint32_t)inner, (cuuint32_t)kTile, (cuuint32_t)Hkv, 1, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUtensorMapDataType dt = kTmaElt == 4   ? CU_TENSOR_MAP_DATA_TYPE_UINT32
                                   : kTmaElt == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                                  : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    CUresult r = fn(map, dt, 5, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D, bool G16, int KV>
cudaError_t launch_typed(const CUtensorMap &km, const CUtensorMap &vm, const Args &a, int grid,
                         int smem, cudaStream_t st) {
    auto kfn = decode_tc_kernel<D, G16, KV>;
    // raise the dynamic shared-memory limit to what this launch needs (per device,
    // only upwards; static shared memory counts against the same per-block budget)
    static int smem_set[64] = {0};  // benign race: idempotent
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    if (dev >= 64 || smem_set[dev] < smem) {
        cudaError_t e =
            cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) smem_set[dev] = smem;
    }
    return launch_pdl(kfn, dim3(grid), dim3(kThreads), smem, st, km, vm, a);
}

}  // namespace tc

namespace tc {
// The plan kernel of one decode call (writes the unit list into the workspace).
cudaError_t launch_plan(const DecodeArgs &d, cudaStream_t st) {
    const DecodePlan &p = d.plan;
    char *ws = static_cast<char *>(d.ws);
    if (p.balanced)
        return launch_pdl(plan_balanced_kernel, dim3(1), dim3(1024), 0, st, d.ctx_lens, d.err,
                          reinterpret_cast<TcHeader *>(ws + p.off_hdr),
                          reinterpret_cast<int32_t *>(ws + p.off_ns),
                          reinterpret_cast<int4 *>(ws + p.off_units),
                          reinterpret_cast<int32_t *>(ws + p.off_cta),
                          reinterpret_cast<int4 *>(ws + p.off_first),
                          reinterpret_cast<long long *>(ws + p.off_starts), d.B, d.MB * d.bs,
                          p.chunk, p.grid, p.sig);
    return launch_pdl(plan_kernel, dim3(1), dim3(1024), 0, st, d.ctx_lens, d.err,
                      reinterpret_cast<TcHeader *>(ws + p.off_hdr),
                      reinterpret_cast<int32_t *>(ws + p.off_ns),
                      reinterpret_cast<int4 *>(ws + p.off_units), d.B, d.MB * d.bs, p.chunk,
                      p.grid * p.units_per_cta, p.sig);
}
}  // namespace tc

cudaError_t launch_decode_plan_only(const DecodeArgs &d, cudaStream_t st) {
    return tc::launch_plan(d, st);
}

cudaError_t launch_decode_tc(const DecodeArgs &d, int kv, cudaStream_t st) {
    using namespace tc;
    const bool int8 = kv != kKvBf16;  // one-byte pools (int8 codes or e4m3)
    const DecodePlan &p = d.plan;
    CUtensorMap km, vm;
    if (!encode_pool_map(&km, d.k_cache, d.N, d.bs, d.Hkv, d.d, d.block_stride, int8) ||
        !encode_pool_map(&vm, d.v_cache, d.N, d.bs, d.Hkv, d.d, d.block_stride, int8))
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
    a.cta_off = reinterpret_cast<const int32_t *>(ws + p.off_cta);
    a.cta_first = reinterpret_cast<const int4 *>(ws + p.off_first);
    a.balanced = p.balanced;
    a.ws_ml = reinterpret_cast<float *>(ws + p.off_ml);
    a.ws_acc = reinterpret_cast<float *>(ws + p.off_acc);
    a.k_scale = d.k_scale;
    a.v_scale = d.v_scale;
    a.ks_off = p.ks_off;
    a.vs_off = p.vs_off;
    a.N = d.N;
    a.B = d.B;
    a.Hq = d.Hq;
    a.Hkv = d.Hkv;
    a.G = d.G;
    a.bs = d.bs;
    a.MB = d.MB;
    a.S = p.S;
    a.nstage = p.nstage;
    a.stage_bytes = p.stage_bytes;
    a.v_off = p.v_off;
    a.box_bytes = d.Hkv * kTile * kBoxRow;
    a.wph = p.wph;
    a.tpw = p.tpw;
    a.n_sub = p.n_sub;
    {
        const int tpb = d.bs / kTile;
        a.tpb_shift = (tpb & (tpb - 1)) == 0 ? __builtin_ctz((unsigned)tpb) : -1;
    }
    a.scale_log2 = d.scale_log2;
    a.sig = p.sig;
    a.sel_ctas = 0;   // the merge launch below adds the selection CTAs when asked
    a.sel_evict = nullptr;
    a.sel_means = nullptr;
    a.sel_scores = nullptr;
    cudaError_t e = cudaSuccess;
    if (!d.reuse_plan) {
        e = launch_plan(d, st);
        if (e != cudaSuccess) return e;
    }
    const bool g16 = d.G > 8;
    if (kv == kKvInt8)  // one-byte pools: d == 128 only (the plan guarantees it)
        e = g16 ? launch_typed<128, true, kKvInt8>(km, vm, a, p.grid, p.smem_bytes, st)
                : launch_typed<128, false, kKvInt8>(km, vm, a, p.grid, p.smem_bytes, st);
    else if (kv == kKvFp8)
        e = g16 ? launch_typed<128, true, kKvFp8>(km, vm, a, p.grid, p.smem_bytes, st)
                : launch_typed<128, false, kKvFp8>(km, vm, a, p.grid, p.smem_bytes, st);
    else if (d.d == 128)
        e = g16 ? launch_typed<128, true, kKvBf16>(km, vm, a, p.grid, p.smem_bytes, st)
                : launch_typed<128, false, kKvBf16>(km, vm, a, p.grid, p.smem_bytes, st);
    else
        e = g16 ? launch_typed<64, true, kKvBf16>(km, vm, a, p.grid, p.smem_bytes, st)
                : launch_typed<64, false, kKvBf16>(km, vm, a, p.grid, p.smem_bytes, st);
    if (e != cudaSuccess) return e;
    bool sel_done = d.sel_evict == nullptr;
    if (p.S > 1 || p.wph > 1) {
        const unsigned rows = (unsigned)((int64_t)d.B * d.Hq);
        // few partials per row (at most (B + P) / B on average with the balanced split,
        // S * wph with an explicit one): a warp per row; many (long contexts of a small
        // batch): a CTA per row, whose warps split the partials
        const int64_t few = 8;
        const bool rows_kernel = p.balanced ? (int64_t)d.B + p.grid <= few * d.B
                                            : (int64_t)p.S * p.wph <= few;
        if (rows_kernel) {
            // the selection, when asked for, takes B CTAs at the front of this launch
            Args am = a;
            if (!sel_done) {
                am.sel_ctas = d.B;
                am.sel_evict = d.sel_evict;
                am.sel_means = d.sel_means;
                am.sel_scores = d.sel_scores;
                sel_done = true;
            }
            const unsigned ctas =
                (rows + kRowsPerMergeCta - 1) / kRowsPerMergeCta + (unsigned)am.sel_ctas;
            const dim3 blk(32 * kRowsPerMergeCta);
            e = d.d == 128 ? launch_pdl(merge_rows_kernel<128>, dim3(ctas), blk, 0, st, am)
                           : launch_pdl(merge_rows_kernel<64>, dim3(ctas), blk, 0, st, am);
        } else {
            e = d.d == 128 ? launch_pdl(merge_tc_kernel<128>, dim3(rows), dim3(128), 0, st, a)
                           : launch_pdl(merge_tc_kernel<64>, dim3(rows), dim3(64), 0, st, a);
        }
    }
    if (e == cudaSuccess && !sel_done)   // no merge launch to carry it: its own kernel
        e = launch_select_pooled(d.sel_evict, d.sel_means, d.sel_scores, d.block_tables,
                                 d.ctx_lens, d.err, d.B, d.MB, d.Hkv, d.bs, d.N, st);
    return e;
}

}  // namespace pkv
