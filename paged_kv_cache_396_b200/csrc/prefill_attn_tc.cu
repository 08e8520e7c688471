// prefill_attn_tc.cu -- multi-query (chunked prefill) paged attention on the
// fifth-generation tensor cores: tcgen05.mma with TMEM accumulators.
//
// Same operation as prefill_attn.cu (t6page.pages.dev "KV cache", "Chunked
// prefill：让 prefill 不阻塞 decode"; "PagedAttention 的算子"): the q_len query
// tokens of a sequence are its last q_len cached tokens and attend causally.
// Used for d = 128 and block sizes that are multiples of 16.
//
// An item = one (sequence, kv head, 256 query rows) as two tiles of 128 rows
// (the MMA M); rows are (query token, head of the GQA group) pairs, so each K/V
// tile serves all G heads of both Q tiles.  Warp roles (320 threads):
//   warps 0-3, 4-7  softmax, one warpgroup per Q tile: thread r owns row r of its
//              tile = TMEM lane r.  Loads its Q row into shared memory per item;
//              per 128-token K/V tile reads its 128 logits from TMEM (four loads,
//              one wait), masks (causal, diagonal tiles only), keeps the running
//              max (lazy: O is rescaled only when the max grows by more than 2^8),
//              writes P = hi + lo (two bf16 parts: the weight's top 16 bits and the
//              remainder's) back over the S columns, and at the end normalises O
//              (or, for a cut item, writes its partial and the last part merges).
//              The per-weight arithmetic runs on packed fp32 pairs: this warp's
//              instruction stream is on the critical path of the tile period.  The two warpgroups work half a step apart, so
//              one computes softmax while the tensor core runs the other tile's
//              products.
//   warp 8     MMA issue (warp-uniform operands, elect.sync picks the issuing
//              lane), in the order PV_A(j), S_A(j+1), PV_B(j), S_B(j+1): S = Q K^T
//              (SS, both K-major) into the tile's S/P columns, O += P_hi V + P_lo V
//              (A from TMEM, V MN-major) into its O columns; completion through
//              tcgen05.commit.  Its lanes also zero the V rows past the context end
//              in a tile that holds them (stale or NaN slots must not meet a zero
//              weight).
//   warp 9     TMA producer: lane p < 8 owns 16-token page p of every tile, looks
//              up its physical block one tile ahead and issues four boxes (K and V,
//              two 64-element slices each).  K and V stages have barriers of their
//              own: a K stage frees when the tile's last S is done, a V stage after
//              its last P V, so the next K tile is on its way about one P V pair
//              earlier than with one barrier per K/V stage.
// TMEM: S/P of tile A at columns [0,128), of tile B at [128,256); O of tile A at
// [256,384), of tile B at [384,512).
// Work: an item is (sequence, kv head, 256 query rows); a segment is a run of one
// item's K/V tiles.  Without a workspace each CTA runs one whole item.  With one
// (balanced mode) a plan kernel ranks the items, then two launches: full waves of
// whole items, and one equal range of the left-over items' tiles per SM, which
// starts as the whole-item CTAs retire (programmatic dependent launch); a segment
// cut from an item leaves fp32 partials that the part finishing last merges (the
// roles of a range CTA walk its segments in a loop, with barrier phases carried
// across segments).
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
constexpr int kKStages = 2;      // K tiles in flight
constexpr int kVStages = 2;      // V tiles in flight
constexpr int kSmem = (2 /*Q x 2*/ + kKStages + kVStages) * kTileB + 1024;
static_assert(kSmem <= 227 * 1024 - 256, "dynamic shared memory above the per-CTA limit");
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

// Two fp32 lanes per instruction (sm_100 packed fp32): each lane rounds as the scalar
// fmaf / addition does.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
// max of three (one instruction on sm_100)
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
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
    uint64_t q_full;              // 256 softmax threads: the segment's Q rows in shared memory
    uint64_t k_full[kKStages];    // TMA bytes of a stage's K tile
    uint64_t v_full[kVStages];    // TMA bytes of a stage's V tile
    uint64_t k_empty[kKStages];   // commit after the last S = Q K^T that read the K tile
    uint64_t v_empty[kVStages];   // commit after the last P V that read the V tile
    uint64_t s_full[2];           // per Q tile: commit after S = Q K^T
    uint64_t p_full[2];           // per Q tile: 128 softmax threads wrote P
    uint64_t pv_done[2];          // per Q tile: commit after O += P V
    uint64_t o_final;             // commit after the last P V of a segment (both tiles)
    uint64_t o_free;              // 256 softmax threads: the segment's O read out of TMEM
    uint32_t tmem_base;
    int abort_flag;
};

// Work items: (sequence b, kv head h, 256-row query tile), dense index
// d = (b * Hkv + h) * X + x, X = ceil(max_q_len / QT), q tile qt = n_qt(b) - 1 - x
// (longest context first); x >= n_qt(b) is no item (no tiles).  A segment is a run
// [jb, je) of one item's K/V tiles.
struct Item {
    int b, h, qt, q0, ql, len, pos0, tok_base, n_kt;   // n_kt = 0: no item or bad length
};

__device__ __forceinline__ Item item_of(const PrefillAttnArgs &a, int d, int X, int QT) {
    Item it;
    const int x = d % X, bh = d / X;
    it.h = bh % a.Hkv;
    it.b = bh / a.Hkv;
    it.q0 = a.cu_q[it.b];
    it.ql = a.cu_q[it.b + 1] - it.q0;
    it.qt = (it.ql + QT - 1) / QT - 1 - x;
    it.len = a.ctx_lens[it.b];
    it.tok_base = it.qt * QT;
    it.pos0 = it.len - it.ql;
    it.n_kt = 0;
    if (it.qt >= 0 && it.len >= 0 && (int64_t)it.len <= (int64_t)a.MB * a.bs && it.ql <= it.len)
        it.n_kt = (it.pos0 + min(it.ql - 1, it.tok_base + QT - 1)) / kN + 1;
    return it;
}

struct Seg {
    int d;        // dense item index; -1: no more segments
    int jb, je;   // K/V tiles of the segment
    int slot;     // partial-result slot; -1: the segment is the whole item
};

// Balanced mode (a plan kernel writes the lists below every call).  With n items
// that have rows and P SMs, the first whole = floor(n / P) P items, in item order,
// run one per CTA (full waves; the CTAs of one (sequence, kv head) sweep its K/V
// together, from L2); the CTAs after those zero the rows of items whose length
// cannot be served.  The r = n - whole items left over are laid end to end (R
// tiles) and CTA k of the second launch takes tiles [k L, (k + 1) L), L =
// ceil(R / P): one or a few segments, the last wave then ends about evenly on
// every SM.  A segment cut from an item writes its partial result to slot 2k (the
// item began in an earlier range) or 2k + 1; for each 32 rows (a softmax warp) the
// part that finishes last merges the item's parts in range order.
struct StreamWs {
    const int *hdr;     // whole, r, R, L, n_bad
    const int *items;   // [n + n_bad] item index by rank, then the bad items
    const int *pre;     // [r + 1] tile offsets of the items left over
    const int *lrank;   // [n_items] rank among the items left over, -1: not left over
    int *cnt;           // [n_items][8] parts done per (item, softmax warp)
    float *part;        // [2P][8 softmax warps][d / 4][32 lanes] float4: O of a part
                        // (not normalised), row = 32 warp + lane
    float *ml;          // [2P][256][2] (m, l) of a part; m in the log2 domain
    int n_items, X, P;
};

__device__ __forceinline__ Seg left_seg(const StreamWs &w, int lr, int k, int R, int L,
                                        int whole) {
    const int a = w.pre[lr], e = w.pre[lr + 1];
    const int r0 = k * L, r1 = min(R, r0 + L);
    Seg s;
    s.d = w.items[whole + lr];
    s.jb = max(a, r0) - a;
    s.je = min(e, r1) - a;
    s.slot = (s.jb == 0 && s.je == e - a) ? -1 : (a < r0 ? 2 * k : 2 * k + 1);
    return s;
}

// Modes.  kGrid: one CTA per item (grid x, y, z = q tile, kv head, sequence).  The
// balanced mode is two launches: kWhole, CTA k runs whole item k of the plan's ranking
// (k < whole), CTA whole + i zeroes the rows of bad-length item i; kLeft, CTA k runs
// the k-th equal range of the left-over items' tiles (one or a few segments, walked in
// a loop by every role).  The whole items keep the loop-free code of the grid mode;
// only the range CTAs carry the segment state.
enum { kGrid = 0, kWhole = 1, kLeft = 2 };
template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_attn_tc_kernel(const __grid_constant__ CUtensorMap km,
                           const __grid_constant__ CUtensorMap vm, const PrefillAttnArgs a,
                           const StreamWs sw) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ Bars bars;
    const int G = a.G, QT = kRows / G;   // query tokens per item (two tiles of 128 rows)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int k = blockIdx.x;
    const int X = kMode != kGrid ? sw.X : (int)gridDim.x;
    // the range launch may start as soon as every whole-item CTA has started (it
    // shares no data with them; it waits for their completion before it exits)
    if constexpr (kMode == kWhole) ptx::grid_launch_dependents();
    auto first_seg = [&]() -> Seg {
        if constexpr (kMode == kWhole) {
            const int whole = sw.hdr[0], n_bad = sw.hdr[4];
            if (k < whole) {
                const int d = sw.items[k];
                return Seg{d, 0, item_of(a, d, X, QT).n_kt, -1};
            }
            if (k - whole < n_bad)   // zero-row CTAs for bad lengths
                return Seg{sw.items[whole + sw.hdr[1] + k - whole], 0, 0, -2};
            return Seg{-1, 0, 0, -1};
        } else if constexpr (kMode == kLeft) {
            const int whole = sw.hdr[0], R = sw.hdr[2], L = sw.hdr[3];
            if (k >= sw.P || k * L >= R) return Seg{-1, 0, 0, -1};
            int lo = 0, hi = sw.hdr[1];   // the left-over item holding tile k L
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (sw.pre[mid] <= k * L) lo = mid;
                else hi = mid;
            }
            return left_seg(sw, lo, k, R, L, whole);
        } else {
            const int d = ((int)blockIdx.z * a.Hkv + (int)blockIdx.y) * X + (int)blockIdx.x;
            const Item it = item_of(a, d, X, QT);
            return Seg{it.n_kt > 0 ? d : -1, 0, it.n_kt, -1};
        }
    };
    auto next_seg = [&](const Seg &cur) -> Seg {
        if constexpr (kMode == kLeft) {
            const int whole = sw.hdr[0], R = sw.hdr[2], L = sw.hdr[3];
            const int lr = sw.lrank[cur.d] + 1;
            if (lr >= sw.hdr[1] || sw.pre[lr] >= min(R, (k + 1) * L)) return Seg{-1, 0, 0, -1};
            return left_seg(sw, lr, k, R, L, whole);
        } else {
            return Seg{-1, 0, 0, -1};
        }
    };
    const Seg seg0 = first_seg();
    // an item whose length cannot be served: zero rows and PA_DEV_BAD_LEN (grid mode:
    // no segment; balanced mode: a listed zero segment, slot -2)
    int bad_d = -1;
    if constexpr (kMode == kGrid) {
        if (seg0.d < 0) bad_d = ((int)blockIdx.z * a.Hkv + (int)blockIdx.y) * X + (int)blockIdx.x;
    } else {
        if (seg0.d < 0) {   // no work for this CTA
            if constexpr (kMode == kLeft) ptx::grid_dependency_wait();
            return;
        }
        if (seg0.slot == -2) bad_d = seg0.d;
    }
    if (bad_d >= 0) {
        const Item it = item_of(a, bad_d, X, QT);
        if (it.qt < 0) return;   // no rows
        if (bad_d % X == 0 && it.h == 0 && tid == 0) raise_flag(a.err, PA_DEV_BAD_LEN);
        for (int r = warp; r < kRows; r += kThreads / 32) {
            const int i = it.tok_base + r / G;
            if (i >= it.ql) continue;
            uint16_t *o = a.out + ((int64_t)(it.q0 + i) * a.Hq + it.h * G + r % G) * kD;
            for (int e = lane; e < kD; e += 32) o[e] = 0;
        }
        return;
    }

    // 1024-byte aligned tiles (the 128-byte swizzle pattern repeats every 1024 bytes)
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    auto sQ = [&](int w) { return base + (uint32_t)(w * kTileB); };
    auto sK = [&](int st) { return base + (uint32_t)((2 + st) * kTileB); };
    auto sV = [&](int st) { return base + (uint32_t)((2 + kKStages + st) * kTileB); };

    // K/V stages start as zeros: a page that is not loaded (bad block id) then
    // holds finite data only
    for (int x = tid; x < (kKStages + kVStages) * kTileB / 16; x += kThreads)
        *reinterpret_cast<uint4 *>(gbase + 2 * kTileB + 16 * x) = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (tid == 0) {
        ptx::mbar_init(&bars.q_full, 256);
        for (int i = 0; i < kKStages; ++i) {
            ptx::mbar_init(&bars.k_full[i], 1);
            ptx::mbar_init(&bars.k_empty[i], 1);
        }
        for (int i = 0; i < kVStages; ++i) {
            ptx::mbar_init(&bars.v_full[i], 1);
            ptx::mbar_init(&bars.v_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&bars.s_full[i], 1);
            ptx::mbar_init(&bars.p_full[i], 128);
            ptx::mbar_init(&bars.pv_done[i], 1);
        }
        ptx::mbar_init(&bars.o_final, 1);
        ptx::mbar_init(&bars.o_free, 256);
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
        const int R = w * 128 + r;               // row of the item
        // Q row of an item -> shared memory, K-major 128-byte swizzle
        auto load_q = [&](const Item &it) {
            const int i = it.tok_base + R / G;
            const uint4 *src = reinterpret_cast<const uint4 *>(
                a.q + ((int64_t)(it.q0 + min(i, it.ql - 1)) * a.Hq + it.h * G + R % G) * kD);
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
        };
        const uint32_t lane_base = tm + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t sbuf = lane_base + w * 128;          // S, then P over it
        const uint32_t obuf = lane_base + kColO + w * 128;  // O
        const float sl = a.scale_log2;
        bool ok = true;
        int jt = 0, sn = 0;   // tiles and segments this CTA has done (barrier phases)
        Seg sg = seg0;
        load_q(item_of(a, sg.d, X, QT));
        while (ok) {
            // what the row needs from its item, taken once (the item itself is not
            // kept live across the tile loop)
            int i, pos, nkt;
            int64_t orow_off;
            {
                const Item it = item_of(a, sg.d, X, QT);
                i = it.tok_base + R / G;             // query token in the sequence's chunk
                pos = it.pos0 + min(i, it.ql - 1);   // causal limit (inclusive)
                orow_off = ((int64_t)(it.q0 + min(i, it.ql - 1)) * a.Hq + it.h * G + R % G) * kD;
                nkt = it.n_kt;
                if (i >= it.ql) i = -1;
            }
            const bool valid = i >= 0;
            float m = -INFINITY, l = 0.f;
            for (int j = sg.jb; j < sg.je && ok; ++j, ++jt) {
                if (!(ok = warp_wait(&bars.s_full[w], jt & 1, abort_flag))) break;
                fence_after();
                // tokens t0 + e with e <= lim are visible to this row (lim >= 127: all)
                const int lim = valid ? pos - j * kN : -1;
                // tiles every row of the warp sees in full (all but the diagonal ones)
                // skip the causal select; with scale > 0 the max is taken on the raw logits
                const bool full = __all_sync(0xffffffffu, lim >= kN - 1) && sl > 0.f;
                // ---- the row's 128 logits of this tile: four 32-column TMEM reads in
                // flight, one wait; then the row maximum of the scaled, masked logits
                // (8 independent max chains, two logits per three-input max)
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
                        for (int e = 0; e < 32; e += 2)
                            mk[(e >> 1) & 7] = max3(mk[(e >> 1) & 7], __uint_as_float(v[c][e]),
                                                    __uint_as_float(v[c][e + 1]));
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
                float mx = max3(max3(mk[0], mk[1], mk[2]), max3(mk[3], mk[4], mk[5]),
                                fmaxf(mk[6], mk[7]));
                if (full) mx *= sl;
                const float mn = fmaxf(m, mx);
                // lazy rescale: a row moves its reference max only when the tile's max
                // exceeds it by more than 8 (weights stay below 2^8 otherwise); the
                // first finite max always moves it (-inf + 8 = -inf)
                const bool move = mn > m + 8.f;
                const bool rescale = move && j > sg.jb && m != -INFINITY;  // O holds tiles
                const float alpha = rescale ? ex2(m - mn) : 1.f;
                if (move) m = mn;
                const float u = m == -INFINITY ? 0.f : m;
                // ---- P = exp2(s - u) as hi + lo bf16 over the S columns: k-step kk
                // (16 tokens) at columns 16kk (hi, 8 columns of bf16 pairs) and 16kk + 8 (lo)
                // (scale-subtract, row sums and the lo remainders two lanes at a time)
                float2 ls[4] = {};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float x[32];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float2 y = fma2(make_float2(__uint_as_float(v[c][e]),
                                                          __uint_as_float(v[c][e + 1])),
                                              make_float2(sl, sl), make_float2(-u, -u));
                        x[e] = y.x;
                        x[e + 1] = y.y;
                    }
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
                            const float2 pp = make_float2(ex2(x[e]), ex2(x[e + 1]));
                            ls[q & 3] = add2(ls[q & 3], pp);
                            // hi = each weight's top 16 bits (truncated), lo = the exact
                            // remainder truncated the same way: hi + lo is within 2^-15 of
                            // the weight, and no conversion instruction runs
                            const uint32_t b0 = __float_as_uint(pp.x), b1 = __float_as_uint(pp.y);
                            wv[16 * half + q] = __byte_perm(b0, b1, 0x7632);
                            const float2 rr = add2(
                                pp, make_float2(__uint_as_float((b0 & 0xffff0000u) ^ 0x80000000u),
                                                __uint_as_float((b1 & 0xffff0000u) ^ 0x80000000u)));
                            wv[16 * half + 8 + q] =
                                __byte_perm(__float_as_uint(rr.x), __float_as_uint(rr.y), 0x7632);
                        }
                    }
                    tmem_st32(sbuf + 32 * c, wv);
                }
                // O is rescaled after P is written, when the logits' registers are free;
                // the P V of this tile is issued only after the arrive below
                if (__any_sync(0xffffffffu, rescale)) {   // warp-collective TMEM access
                    if (!(ok = warp_wait(&bars.pv_done[w], (jt - 1) & 1, abort_flag))) break;
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
                const float2 ls2 = add2(add2(ls[0], ls[1]), add2(ls[2], ls[3]));
                l = l * alpha + (ls2.x + ls2.y);
                tmem_wait_st();
                fence_before();
                ptx::mbar_arrive(&bars.p_full[w]);
            }
            if (!ok) break;
            // every S of this segment is done: the next segment's Q rows can go to
            // shared memory now, so its first S overlaps this epilogue
            const Seg nx = next_seg(sg);
            if (nx.d >= 0) load_q(item_of(a, nx.d, X, QT));
            if (!(ok = warp_wait(&bars.o_final, sn & 1, abort_flag))) break;
            fence_after();
            if (sg.slot < 0) {   // the whole item: the normalised bf16 output row
                const float inv = l > 0.f ? 1.f / l : 0.f;
                uint4 *orow = reinterpret_cast<uint4 *>(a.out + orow_off);
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
                            for (int q = 0; q < 4; ++q) {
                                const int e = 4 * e4 + q;
                                w4[q] = (uint32_t)f32_to_bf16_rn(__uint_as_float(v[2 * e]) * inv) |
                                        ((uint32_t)f32_to_bf16_rn(__uint_as_float(v[2 * e + 1]) *
                                                                  inv)
                                         << 16);
                            }
                            orow[4 * c + e4] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        }
                    }
                }
            } else {   // a part of the item: its partial result, then the merge
                // the item's parts: ranges k0 .. k1 of the left-over tiles
                const int L = sw.hdr[3];
                const int a0 = sw.pre[sw.lrank[sg.d]];
                const int k0 = a0 / L, k1 = (a0 + nkt - 1) / L;
                auto slot_of = [&](int kk) { return a0 < kk * L ? 2 * kk : 2 * kk + 1; };
                // [slot][softmax warp][d/4][lane] float4: each warp store covers 512
                // contiguous bytes
                float4 *pw = reinterpret_cast<float4 *>(sw.part) +
                             ((int64_t)sg.slot * 8 + warp) * (kD / 4) * 32 + lane;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t v[32];
                    tmem_ld32(obuf + 32 * c, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4)
                        pw[(8 * c + e4) * 32] = make_float4(
                            __uint_as_float(v[4 * e4]), __uint_as_float(v[4 * e4 + 1]),
                            __uint_as_float(v[4 * e4 + 2]), __uint_as_float(v[4 * e4 + 3]));
                }
                if (valid)
                    *reinterpret_cast<float2 *>(sw.ml + ((int64_t)sg.slot * kRows + R) * 2) =
                        make_float2(m, l);
                // the warp whose part completes its 32 rows' set merges them: a
                // counter per (item, softmax warp), zeroed by the plan kernel
                __threadfence();
                __syncwarp();
                int last = 0;
                if (lane == 0)
                    last = atomicAdd(sw.cnt + (int64_t)sg.d * 8 + warp, 1) == k1 - k0;
                if (__shfl_sync(0xffffffffu, last, 0)) {
                    __threadfence();
                    // M = max m_c, out = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c over
                    // the item's parts in range order; the part rows' loads are issued
                    // 16 at a time (two parts x 32 dims)
                    auto mlrow = [&](int kk) {
                        return __ldcg(reinterpret_cast<const float2 *>(
                            sw.ml + ((int64_t)slot_of(kk) * kRows + R) * 2));
                    };
                    // M and L in one pass: L rescaled whenever M grows
                    float M = -INFINITY, Ls = 0.f;
#pragma unroll 4
                    for (int kk = k0; kk <= k1; ++kk) {
                        const float2 ml = mlrow(kk);
                        if (ml.x == -INFINITY) continue;
                        if (ml.x > M) {
                            Ls = Ls * exp2f(M - ml.x);   // exp2(-inf) = 0 for the first
                            M = ml.x;
                        }
                        Ls = fmaf(ml.y, exp2f(ml.x - M), Ls);
                    }
                    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
                    uint4 *orow = reinterpret_cast<uint4 *>(a.out + orow_off);
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {   // 32 dims a chunk
                        float acc[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) acc[e] = 0.f;
                        auto add = [&](const float4 (&x)[8], float f) {
#pragma unroll
                            for (int e4 = 0; e4 < 8; ++e4) {
                                acc[4 * e4] = fmaf(x[e4].x, f, acc[4 * e4]);
                                acc[4 * e4 + 1] = fmaf(x[e4].y, f, acc[4 * e4 + 1]);
                                acc[4 * e4 + 2] = fmaf(x[e4].z, f, acc[4 * e4 + 2]);
                                acc[4 * e4 + 3] = fmaf(x[e4].w, f, acc[4 * e4 + 3]);
                            }
                        };
                        auto load = [&](int kk, float4 (&x)[8]) {
                            const float4 *src = reinterpret_cast<const float4 *>(sw.part) +
                                                ((int64_t)slot_of(kk) * 8 + warp) * (kD / 4) * 32 +
                                                (8 * c) * 32 + lane;
#pragma unroll
                            for (int e4 = 0; e4 < 8; ++e4) x[e4] = __ldcg(src + 32 * e4);
                        };
                        if (M != -INFINITY) {
                            int kk = k0;
                            for (; kk + 1 <= k1; kk += 2) {
                                float4 x0[8], x1[8];
                                load(kk, x0);
                                load(kk + 1, x1);
                                add(x0, exp2f(mlrow(kk).x - M));
                                add(x1, exp2f(mlrow(kk + 1).x - M));
                            }
                            if (kk <= k1) {
                                float4 x0[8];
                                load(kk, x0);
                                add(x0, exp2f(mlrow(kk).x - M));
                            }
                        }
                        if (valid) {
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4)
                                orow[4 * c + q4] = make_uint4(
                                    (uint32_t)f32_to_bf16_rn(acc[8 * q4] * inv) |
                                        ((uint32_t)f32_to_bf16_rn(acc[8 * q4 + 1] * inv) << 16),
                                    (uint32_t)f32_to_bf16_rn(acc[8 * q4 + 2] * inv) |
                                        ((uint32_t)f32_to_bf16_rn(acc[8 * q4 + 3] * inv) << 16),
                                    (uint32_t)f32_to_bf16_rn(acc[8 * q4 + 4] * inv) |
                                        ((uint32_t)f32_to_bf16_rn(acc[8 * q4 + 5] * inv) << 16),
                                    (uint32_t)f32_to_bf16_rn(acc[8 * q4 + 6] * inv) |
                                        ((uint32_t)f32_to_bf16_rn(acc[8 * q4 + 7] * inv) << 16));
                        }
                    }
                }
            }
            fence_before();
            ptx::mbar_arrive(&bars.o_free);
            ++sn;
            if (nx.d < 0) break;
            sg = nx;
        }
    } else if (warp == 8) {
        // ======================= MMA issue =======================
        // tensor-core order per K/V tile j: PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so
        // each softmax warpgroup works while the other tile's products run
        const uint32_t id_qk = idesc(false), id_pv = idesc(true);
        auto zero_tail = [&](int j, int st, int len) {
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
        // jj: tile index within the segment (0: O starts afresh)
        auto issue_pv = [&](int w, int jj, int st) {
#pragma unroll
            for (int kk = 0; kk < kN / 16; ++kk) {
                // V: 16 token rows per k-step; N = 128 dims across the two slices
                const uint64_t vd = sdesc(sV(st) + (uint32_t)(kk * 16 * 128), kSlice, 1024);
                mma_ts(tm + kColO + w * 128, tm + w * 128 + 16 * kk, vd, id_pv,
                       (jj > 0 || kk > 0) ? 1u : 0u);
                mma_ts(tm + kColO + w * 128, tm + w * 128 + 16 * kk + 8, vd, id_pv, 1u);
            }
            commit(&bars.pv_done[w]);
        };
        bool ok = true;
        int jt = 0, sn = 0;
        for (Seg sg = seg0; sg.d >= 0 && ok; sg = next_seg(sg), ++sn) {
            const int len = a.ctx_lens[item_of(a, sg.d, X, QT).b];
            const int nt = sg.je - sg.jb;
            if (!(ok = warp_wait(&bars.q_full, sn & 1, abort_flag) &&
                       warp_wait(&bars.k_full[jt % kKStages], (jt / kKStages) & 1, abort_flag)))
                break;
            // the new S overwrites the columns the previous segment's last P V read P
            // from: that segment's products are complete first
            if (sn > 0 && !(ok = warp_wait(&bars.o_final, (sn - 1) & 1, abort_flag))) break;
            fence_after();
            issue_s(0, jt % kKStages);
            issue_s(1, jt % kKStages);
            commit(&bars.k_empty[jt % kKStages]);
            for (int jj = 0; jj < nt && ok; ++jj, ++jt) {
                const int st = jt % kVStages, st1 = (jt + 1) % kKStages;
                const bool more = jj + 1 < nt;
                // ---- tile A
                if (!(ok = warp_wait(&bars.p_full[0], jt & 1, abort_flag))) break;
                if (jj == 0 && sn > 0 &&   // O of the previous segment is read out
                    !(ok = warp_wait(&bars.o_free, (sn - 1) & 1, abort_flag)))
                    break;
                if (!(ok = warp_wait(&bars.v_full[st], (jt / kVStages) & 1, abort_flag))) break;
                zero_tail(sg.jb + jj, st, len);
                fence_after();
                issue_pv(0, jj, st);
                if (more) {
                    if (!(ok = warp_wait(&bars.k_full[st1], ((jt + 1) / kKStages) & 1,
                                         abort_flag)))
                        break;
                    // S_A(j+1) overwrites the columns PV_A(j) reads its P from
                    if (!(ok = warp_wait(&bars.pv_done[0], jt & 1, abort_flag))) break;
                    fence_after();
                    issue_s(0, st1);
                }
                // ---- tile B
                if (!(ok = warp_wait(&bars.p_full[1], jt & 1, abort_flag))) break;
                fence_after();
                issue_pv(1, jj, st);
                commit(&bars.v_empty[st]);
                if (!more) commit(&bars.o_final);
                if (more) {
                    if (!(ok = warp_wait(&bars.pv_done[1], jt & 1, abort_flag))) break;
                    fence_after();
                    issue_s(1, st1);
                    commit(&bars.k_empty[st1]);
                }
            }
        }
    } else {
        // ======================= TMA producer (warp 9) =======================
        // lane pg < 8 owns 16-token page pg of every tile: it looks up the page's
        // physical block (one tile ahead, so the table read is off the critical
        // path) and issues the page's four boxes
        bool ok = true;
        int jt = 0;
        for (Seg sg = seg0; sg.d >= 0 && ok; sg = next_seg(sg)) {
            const Item it = item_of(a, sg.d, X, QT);
            const int32_t *btr = a.block_tables + (int64_t)it.b * a.MB;
            auto lookup = [&](int j) -> int32_t {
                const int t = j * kN + 16 * lane;
                return (lane < kN / 16 && t < it.len) ? btr[t / a.bs] : -1;
            };
            int32_t next = lookup(sg.jb);
            for (int j = sg.jb; j < sg.je && ok; ++j, ++jt) {
                const int32_t blk = next;
                if (j + 1 < sg.je) next = lookup(j + 1);
                const int t = j * kN + 16 * lane;
                const bool in = lane < kN / 16 && t < it.len;
                // pages inside the context with a valid block id are loaded; the others
                // are not (their rows are masked, and V rows past the end zeroed)
                const bool load = in && blk >= 0 && (int64_t)blk < a.N;
                if (in && !load) raise_flag(a.err, PA_DEV_BAD_BLOCK);
                const unsigned lm = __ballot_sync(0xffffffffu, load);
                const int off = t % a.bs;
                // K first: its stage frees when the tile's last S is done, well before
                // the V stage (after the last P V)
#pragma unroll
                for (int kv = 0; kv < 2; ++kv) {
                    const int ns = kv ? kVStages : kKStages, st = jt % ns;
                    uint64_t *full = kv ? &bars.v_full[st] : &bars.k_full[st];
                    uint64_t *empty = kv ? &bars.v_empty[st] : &bars.k_empty[st];
                    if (jt >= ns && !(ok = warp_wait(empty, ((jt / ns) - 1) & 1, abort_flag)))
                        break;
                    if (lane == 0)
                        ptx::mbar_arrive_expect_tx(full, (uint32_t)__popc(lm) * 2u * 2048u);
                    __syncwarp();
                    if (load) {
                        const CUtensorMap *map = kv ? &vm : &km;
                        const uint32_t s0 = kv ? sV(st) : sK(st);
#pragma unroll
                        for (int sl = 0; sl < 2; ++sl) {
                            const uint32_t dst = s0 + (uint32_t)(sl * kSlice + lane * 16 * 128);
                            ptx::tma_load_5d(gbase + (dst - base), map, full, 0, off, it.h, sl,
                                             blk);
                        }
                    }
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
    // the call is complete only when the whole-item launch is
    if constexpr (kMode == kLeft) ptx::grid_dependency_wait();
}

// Exclusive prefix sum over the 1024 threads of a CTA; *total receives the sum.
__device__ __forceinline__ int cta_scan(int v, int *total) {
    __shared__ int s_w[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) s_w[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int x = s_w[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        s_w[lane] = x;   // inclusive totals of warps 0..lane
    }
    __syncthreads();
    const int before = warp ? s_w[warp - 1] : 0;
    *total = s_w[31];
    __syncthreads();
    return before + inc - v;
}

// Balanced mode, before the attention kernel (one CTA of 1024 threads): the item
// ranks, the tile offsets of the items left over, L, zeroed merge counters.
__global__ void __launch_bounds__(1024) prefill_plan_kernel(const PrefillAttnArgs a,
                                                            const StreamWs sw) {
    constexpr int kCache = 4096;   // items whose tile counts are kept in shared memory
    __shared__ int s_nk[kCache];
    const int tid = threadIdx.x;
    const int QT = kRows / a.G, X = sw.X, n_items = sw.n_items, P = sw.P;
    int *hdr = const_cast<int *>(sw.hdr);
    int *items = const_cast<int *>(sw.items);
    int *pre = const_cast<int *>(sw.pre);
    int *lrank = const_cast<int *>(sw.lrank);
    for (int x = tid; x < n_items * 8; x += 1024) sw.cnt[x] = 0;
    // tile count of item d, or -1 when the item has rows but a bad length
    auto tiles = [&](int d) -> int {
        if (d < kCache) return s_nk[d];
        const Item it = item_of(a, d, X, QT);
        return it.n_kt > 0 ? it.n_kt : (it.qt >= 0 ? -1 : 0);
    };
    for (int d = tid; d < min(n_items, kCache); d += 1024) {
        const Item it = item_of(a, d, X, QT);
        s_nk[d] = it.n_kt > 0 ? it.n_kt : (it.qt >= 0 ? -1 : 0);
    }
    __syncthreads();
    int n = 0;
    for (int b0 = 0; b0 < n_items; b0 += 1024) {
        const int d = b0 + tid;
        int t;
        cta_scan(d < n_items && tiles(d) > 0, &t);
        n += t;
    }
    const int whole = n / P * P;
    int rank0 = 0, bad0 = 0, R = 0;
    for (int b0 = 0; b0 < n_items; b0 += 1024) {
        const int d = b0 + tid;
        const int nk = d < n_items ? tiles(d) : 0;
        int t;
        const int rank = rank0 + cta_scan(nk > 0, &t);
        rank0 += t;
        const int bad = bad0 + cta_scan(nk < 0, &t);
        bad0 += t;
        const bool left = nk > 0 && rank >= whole;
        const int off = R + cta_scan(left ? nk : 0, &t);
        R += t;
        if (nk > 0) items[rank] = d;
        if (nk < 0) items[n + bad] = d;
        if (left) pre[rank - whole] = off;
        if (d < n_items) lrank[d] = left ? rank - whole : -1;
    }
    if (tid == 0) {
        pre[n - whole] = R;
        hdr[0] = whole;
        hdr[1] = n - whole;
        hdr[2] = R;
        hdr[3] = R > 0 ? (R + P - 1) / P : 1;
        hdr[4] = bad0;
    }
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

namespace {
inline size_t up256(size_t x) { return (x + 255) / 256 * 256; }
struct StreamLayout {
    int64_t n_items;
    int X;
    size_t off_items, off_pre, off_lrank, off_cnt, off_part, off_ml, total;
};
// header | item ranks | left-over tile offsets | left-over ranks | merge counters |
// partial results of at most 2P parts
StreamLayout stream_layout(int B, int Hkv, int G, int max_q_len, int sms) {
    StreamLayout L;
    const int QT = kRows / G;
    L.X = (max_q_len + QT - 1) / QT;
    L.n_items = (int64_t)B * Hkv * L.X;
    L.off_items = 256;
    L.off_pre = L.off_items + up256((size_t)L.n_items * 4);
    L.off_lrank = L.off_pre + up256((size_t)(L.n_items + 1) * 4);
    L.off_cnt = L.off_lrank + up256((size_t)L.n_items * 4);
    L.off_part = L.off_cnt + up256((size_t)L.n_items * 8 * 4);
    L.off_ml = L.off_part + up256((size_t)2 * sms * kRows * kD * 4);
    L.total = L.off_ml + up256((size_t)2 * sms * kRows * 2 * 4);
    return L;
}
}  // namespace

size_t prefill_attn_tc_workspace_bytes(const PrefillAttnArgs &a, int max_q_len, int sms) {
    if (!prefill_attn_tc_supported(a) || max_q_len <= 0 || a.B <= 0) return 0;
    const StreamLayout L = stream_layout(a.B, a.Hkv, a.G, max_q_len, sms);
    if (L.n_items + 1 > INT32_MAX) return 0;
    return L.total;
}

cudaError_t launch_prefill_attn_tc(const PrefillAttnArgs &a, int max_q_len, void *ws,
                                   size_t ws_bytes, int sms, cudaStream_t st) {
    CUtensorMap km, vm;
    if (!encode_head_map(&km, a.k_cache, a.N, a.bs, a.Hkv, a.block_stride) ||
        !encode_head_map(&vm, a.v_cache, a.N, a.bs, a.Hkv, a.block_stride))
        return cudaErrorInvalidValue;
    const size_t need = prefill_attn_tc_workspace_bytes(a, max_q_len, sms);
    const bool stream = ws != nullptr && need > 0 && ws_bytes >= need;
    static bool attr_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    if (dev >= 64 || !attr_set[dev]) {
        for (auto kfn : {prefill_attn_tc_kernel<kGrid>, prefill_attn_tc_kernel<kWhole>,
                         prefill_attn_tc_kernel<kLeft>}) {
            cudaError_t e =
                cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
            if (e != cudaSuccess) return e;
        }
        if (dev < 64) attr_set[dev] = true;
    }
    StreamWs sw = {};
    if (!stream) {
        const int QT = kRows / a.G;
        dim3 grid((unsigned)((max_q_len + QT - 1) / QT), (unsigned)a.Hkv, (unsigned)a.B);
        prefill_attn_tc_kernel<kGrid><<<grid, kThreads, kSmem, st>>>(km, vm, a, sw);
        return cudaGetLastError();
    }
    // balanced: plan; the whole items and the zero-row CTAs; one range of the left-over
    // tiles per SM, launched to start as the whole-item CTAs retire (cut items are
    // merged by their last part)
    const StreamLayout L = stream_layout(a.B, a.Hkv, a.G, max_q_len, sms);
    char *w = static_cast<char *>(ws);
    sw.hdr = reinterpret_cast<int *>(w);
    sw.items = reinterpret_cast<int *>(w + L.off_items);
    sw.pre = reinterpret_cast<int *>(w + L.off_pre);
    sw.lrank = reinterpret_cast<int *>(w + L.off_lrank);
    sw.cnt = reinterpret_cast<int *>(w + L.off_cnt);
    sw.part = reinterpret_cast<float *>(w + L.off_part);
    sw.ml = reinterpret_cast<float *>(w + L.off_ml);
    sw.n_items = (int)L.n_items;
    sw.X = L.X;
    sw.P = sms;
    prefill_plan_kernel<<<1, 1024, 0, st>>>(a, sw);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // whole + n_bad <= n_items CTAs do work; the rest return at once
    prefill_attn_tc_kernel<kWhole><<<(unsigned)L.n_items, kThreads, kSmem, st>>>(km, vm, a, sw);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)sms);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_attn_tc_kernel<kLeft>, km, vm, a, sw);
}

}  // namespace pkv
