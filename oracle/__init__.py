"""fp64 CPU oracle for paged decode attention (ctypes wrapper over oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()`` and
by the CPU-baseline leg of ``bench.py``; never by the library.  It shares no code
with the CUDA path.  Every function takes and returns numpy arrays on the host;
bf16 tensors travel as their uint16 bit patterns.

Pages cited (by title and section):
  [KVL]  blog.hotdry.top "KV缓存内存布局优化" -- PagedAttention paging, PagedEviction.
  [VKV]  ybb.press "LLM 推理 KV Cache 内存管理深度工程实践" -- §2.1 BlockTable,
         §2.2 paged_attention_forward, §6.1 INT8 quantiser, §6.2 GQA.
  [NANO] blog.hotdry.top nano-vLLM KV cache -- physical layout [2, L, N, bs, n_kv, d].
  [KVP]  t6page.pages.dev "KV cache" -- eq. kv-per-token, eq. kv-llama3-8b,
         table tbl-kv-llama3-context, "PagedAttention 的算子".
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        # ORACLE_LIB names another build of oracle.c; tests/oracle_mutants.py uses it
        # to load copies with one planted mistake each
        path = os.environ.get("ORACLE_LIB") or _build.build()
        lib = ctypes.CDLL(path)
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        p = ctypes.c_void_p
        lib.or_kv_bytes_per_token.restype = i64
        lib.or_kv_bytes_per_token.argtypes = [i64, i64, i64, i64]
        lib.or_num_blocks.restype = i64
        lib.or_num_blocks.argtypes = [i64, i64]
        lib.or_slot.restype = i64
        lib.or_slot.argtypes = [p, i64, i64]
        lib.or_append_kv.restype = None
        lib.or_append_kv.argtypes = [p, p, p, p, i64, p, i32, p, i32, i32, i32, i32, i32, p]
        lib.or_append_kv_int8.restype = None
        lib.or_append_kv_int8.argtypes = [p, p, p, p, p, p, i64, p, i32, p, i32, i32, i32, i32,
                                          i32, p]
        lib.or_paged_decode.restype = None
        lib.or_paged_decode.argtypes = [p, p, p, p, i64, p, i32, p, i32, i32, i32, i32, i32, dbl]
        lib.or_paged_decode_int8.restype = None
        lib.or_paged_decode_int8.argtypes = [p, p, p, p, p, p, i64, p, i32, p, i32, i32, i32, i32,
                                             i32, dbl]
        lib.or_score_tokens.restype = None
        lib.or_score_tokens.argtypes = [p, p, p, i64, p, i32, p, i32, i32, i32, i32]
        lib.or_score_tokens_int8.restype = None
        lib.or_score_tokens_int8.argtypes = [p, p, p, p, p, i64, p, i32, p, i32, i32, i32, i32]
        lib.or_select_evict_block.restype = None
        lib.or_select_evict_block.argtypes = [p, p, p, p, p, i32, i32, i32, i32]
        lib.or_quantize_int8.restype = None
        lib.or_quantize_int8.argtypes = [p, i64, i32, p, p]
        lib.or_quantize_e4m3.restype = None
        lib.or_quantize_e4m3.argtypes = [p, i64, p]
        lib.or_prefill_scores.restype = None
        lib.or_prefill_scores.argtypes = [p, p, p, i64, i32, i32]
        lib.or_prefill_select.restype = None
        lib.or_prefill_select.argtypes = [p, p, p, p, i32, i32]
        lib.or_prefill_pack.restype = None
        lib.or_prefill_pack.argtypes = [p, p, p, p, p, i32, p, p, i64, p, i32, i32, i32, i32, i32]
        lib.or_evict_compact.restype = None
        lib.or_evict_compact.argtypes = [p, p, p, p, i32, i32, i32]
        lib.or_select_evict_threshold.restype = None
        lib.or_select_evict_threshold.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i64, i64,
                                                  dbl, dbl]
        lib.or_evict_compact_mask.restype = None
        lib.or_evict_compact_mask.argtypes = [p, p, p, p, i32, i32, i32]
        lib.or_paged_prefill.restype = None
        lib.or_paged_prefill.argtypes = [p, p, p, p, p, i64, p, i32, p, i32, i32, i32, i32, i32,
                                         dbl]
        lib.or_set_threads.restype = None
        lib.or_set_threads.argtypes = [i32]
        lib.or_e4m3_to_f64.restype = dbl
        lib.or_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.or_append_kv_fp8.restype = None
        lib.or_append_kv_fp8.argtypes = [p, p, p, p, i64, p, i32, p, i32, i32, i32, i32, i32, p]
        lib.or_paged_decode_fp8.restype = None
        lib.or_paged_decode_fp8.argtypes = [p, p, p, p, i64, p, i32, p, i32, i32, i32, i32, i32,
                                            dbl]
        _LIB = lib
    return _LIB


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


_THREADS = None


def threads() -> int:
    """OpenMP threads the oracle's parallel loops use (set_threads, else
    OMP_NUM_THREADS, else all cores)."""
    if _THREADS is not None:
        return _THREADS
    env = os.environ.get("OMP_NUM_THREADS")
    return int(env) if env else (os.cpu_count() or 1)


def set_threads(n: int) -> None:
    """Use n OpenMP threads from now on (timing only: results do not depend on it)."""
    global _THREADS
    _lib().or_set_threads(int(n))
    _THREADS = int(n)


# --------------------------------------------------------------------------- sizes
def kv_bytes_per_token(L: int, n_kv: int, d: int, elt_bytes: int) -> int:
    """2 * L * n_kv * d * bytes ([KVP] eq. kv-per-token; [VKV] §1)."""
    return int(_lib().or_kv_bytes_per_token(L, n_kv, d, elt_bytes))


def num_blocks(length: int, bs: int) -> int:
    """ceil(len / bs) blocks ([VKV] §2.1 allocate, §2.2 loop bound)."""
    return int(_lib().or_num_blocks(length, bs))


def slot(bt_row: np.ndarray, pos: int, bs: int) -> int:
    """bt[pos // bs] * bs + pos % bs ([VKV] §2.1 append_slot)."""
    row = _c(bt_row, np.int32)
    return int(_lib().or_slot(_ptr(row), pos, bs))


# --------------------------------------------------------------------------- append
def append_kv(k_new, v_new, k_cache, v_cache, block_stride, bt, positions, bs):
    """In-place append of k_new/v_new [B, n_new, Hkv, d] (uint16 bf16 bits) into the
    pools (flat uint16 arrays, modified).  Returns slots [B, n_new] int64."""
    k_new = _c(k_new, np.uint16)
    v_new = _c(v_new, np.uint16)
    bt = _c(bt, np.int32)
    positions = _c(positions, np.int32)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    B, n_new, Hkv, d = k_new.shape
    slots = np.empty((B, n_new), np.int64)
    _lib().or_append_kv(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), block_stride,
                        _ptr(bt), bt.shape[1], _ptr(positions), B, n_new, Hkv, d, bs, _ptr(slots))
    return slots


def append_kv_int8(k_new, v_new, kq, vq, k_scale, v_scale, block_stride, bt, positions, bs):
    """INT8 append: quantise ([VKV] §6.1, fp32) and store codes/scales in place."""
    k_new = _c(k_new, np.uint16)
    v_new = _c(v_new, np.uint16)
    bt = _c(bt, np.int32)
    positions = _c(positions, np.int32)
    for a in (kq, vq, k_scale, v_scale):
        assert a.flags.c_contiguous
    B, n_new, Hkv, d = k_new.shape
    slots = np.empty((B, n_new), np.int64)
    _lib().or_append_kv_int8(_ptr(k_new), _ptr(v_new), _ptr(kq), _ptr(vq), _ptr(k_scale),
                             _ptr(v_scale), block_stride, _ptr(bt), bt.shape[1], _ptr(positions),
                             B, n_new, Hkv, d, bs, _ptr(slots))
    return slots


# --------------------------------------------------------------------------- attention
def paged_decode(q, k_cache, v_cache, block_stride, bt, ctx_lens, Hkv, bs, scale):
    """fp64 paged decode attention.  q [B, Hq, d] uint16 (bf16 bits); pools flat
    uint16; bt [B, MB] int32; ctx_lens [B] int32.  Returns out [B, Hq, d] float64.
    [VKV] §2.2 paged_attention_forward; [KVP] "PagedAttention 的算子"."""
    q = _c(q, np.uint16)
    k_cache = _c(k_cache, np.uint16)
    v_cache = _c(v_cache, np.uint16)
    bt = _c(bt, np.int32)
    ctx_lens = _c(ctx_lens, np.int32)
    B, Hq, d = q.shape
    out = np.empty((B, Hq, d), np.float64)
    _lib().or_paged_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), block_stride,
                           _ptr(bt), bt.shape[1], _ptr(ctx_lens), B, Hq, Hkv, d, bs, scale)
    return out


def paged_decode_int8(q, kq, vq, k_scale, v_scale, block_stride, bt, ctx_lens, Hkv, bs, scale):
    """fp64 paged decode over an INT8 pool dequantised as scale * code ([VKV] §6.1)."""
    q = _c(q, np.uint16)
    kq = _c(kq, np.int8)
    vq = _c(vq, np.int8)
    k_scale = _c(k_scale, np.float32)
    v_scale = _c(v_scale, np.float32)
    bt = _c(bt, np.int32)
    ctx_lens = _c(ctx_lens, np.int32)
    B, Hq, d = q.shape
    out = np.empty((B, Hq, d), np.float64)
    _lib().or_paged_decode_int8(_ptr(out), _ptr(q), _ptr(kq), _ptr(vq), _ptr(k_scale),
                                _ptr(v_scale), block_stride, _ptr(bt), bt.shape[1],
                                _ptr(ctx_lens), B, Hq, Hkv, d, bs, scale)
    return out


# --------------------------------------------------------------------------- eviction
def score_tokens(k_cache, v_cache, block_stride, bt, ctx_lens, Hkv, d, bs):
    """S = ||V|| / ||K|| per (token, kv head) ([KVL] PagedEviction).  Returns
    scores [B, MB*bs, Hkv] float64 with NaN where t >= len_b."""
    k_cache = _c(k_cache, np.uint16)
    v_cache = _c(v_cache, np.uint16)
    bt = _c(bt, np.int32)
    ctx_lens = _c(ctx_lens, np.int32)
    B, MB = bt.shape
    scores = np.full((B, MB * bs, Hkv), np.nan, np.float64)
    _lib().or_score_tokens(_ptr(scores), _ptr(k_cache), _ptr(v_cache), block_stride, _ptr(bt),
                           MB, _ptr(ctx_lens), B, Hkv, d, bs)
    return scores


def score_tokens_int8(kq, vq, k_scale, v_scale, block_stride, bt, ctx_lens, Hkv, d, bs):
    """Norm-ratio score over dequantised INT8 values."""
    kq = _c(kq, np.int8)
    vq = _c(vq, np.int8)
    k_scale = _c(k_scale, np.float32)
    v_scale = _c(v_scale, np.float32)
    bt = _c(bt, np.int32)
    ctx_lens = _c(ctx_lens, np.int32)
    B, MB = bt.shape
    scores = np.full((B, MB * bs, Hkv), np.nan, np.float64)
    _lib().or_score_tokens_int8(_ptr(scores), _ptr(kq), _ptr(vq), _ptr(k_scale), _ptr(v_scale),
                                block_stride, _ptr(bt), MB, _ptr(ctx_lens), B, Hkv, d, bs)
    return scores


def select_evict_block(scores, ctx_lens, bs):
    """Lowest-mean full block per sequence ([KVL] PagedEviction, decode phase).
    scores [B, MB*bs, Hkv] (any float dtype; widened to fp64, exact for fp32).
    Returns (evict [B] int32, means [B, MB] float64 (NaN = not a candidate),
    gap [B] float64 = second-lowest minus lowest mean)."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    ctx_lens = _c(ctx_lens, np.int32)
    B, T, Hkv = scores.shape
    MB = T // bs
    evict = np.empty(B, np.int32)
    means = np.empty((B, MB), np.float64)
    gap = np.empty(B, np.float64)
    _lib().or_select_evict_block(_ptr(evict), _ptr(means), _ptr(gap), _ptr(scores),
                                 _ptr(ctx_lens), B, MB, Hkv, bs)
    return evict, means, gap


# --------------------------------------------------------------------------- int8
def quantize_int8(x):
    """fp32 mirror of [VKV] §6.1: rows of d bf16 values -> (codes int8, scales float32)."""
    x = _c(x, np.uint16)
    d = x.shape[-1]
    rows = x.size // d
    codes = np.empty(x.shape, np.int8)
    scales = np.empty(x.shape[:-1], np.float32)
    _lib().or_quantize_int8(_ptr(x), rows, d, _ptr(codes), _ptr(scales))
    return codes, scales


# --------------------------------------------------------------------------- fp8
def quantize_e4m3(x):
    """bf16 bits -> e4m3 codes (uint8), round to nearest even, saturating at 448
    ([VKV] §6.1 FP8 branch: cast to float8_e4m3fn)."""
    x = _c(x, np.uint16)
    codes = np.empty(x.shape, np.uint8)
    _lib().or_quantize_e4m3(_ptr(x), x.size, _ptr(codes))
    return codes


def e4m3_values(codes):
    """Exact values of e4m3 codes as float64."""
    codes = np.asarray(codes, np.uint8)
    f = _lib().or_e4m3_to_f64
    return np.vectorize(lambda c: f(int(c)), otypes=[np.float64])(codes)


def append_kv_fp8(k_new, v_new, k_cache, v_cache, block_stride, bt, positions, bs):
    """FP8 append in place (pools: flat uint8 e4m3 codes).  Returns slots."""
    k_new = _c(k_new, np.uint16)
    v_new = _c(v_new, np.uint16)
    bt = _c(bt, np.int32)
    positions = _c(positions, np.int32)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    B, n_new, Hkv, d = k_new.shape
    slots = np.empty((B, n_new), np.int64)
    _lib().or_append_kv_fp8(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), block_stride,
                            _ptr(bt), bt.shape[1], _ptr(positions), B, n_new, Hkv, d, bs,
                            _ptr(slots))
    return slots


def paged_decode_fp8(q, k_cache, v_cache, block_stride, bt, ctx_lens, Hkv, bs, scale):
    """fp64 paged decode over e4m3 pools (codes decoded exactly)."""
    q = _c(q, np.uint16)
    k_cache = _c(k_cache, np.uint8)
    v_cache = _c(v_cache, np.uint8)
    bt = _c(bt, np.int32)
    ctx_lens = _c(ctx_lens, np.int32)
    B, Hq, d = q.shape
    out = np.empty((B, Hq, d), np.float64)
    _lib().or_paged_decode_fp8(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), block_stride,
                               _ptr(bt), bt.shape[1], _ptr(ctx_lens), B, Hq, Hkv, d, bs, scale)
    return out


# --------------------------------------------------------------------------- prefill stage
def prefill_scores(k, v):
    """Token importance at prefill ([KVL] PagedEviction two-stage strategy): the
    mean over kv heads of ||V||/||K||.  k, v [T, Hkv, d] bf16 bits -> [T] float64."""
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    T, Hkv, d = k.shape
    scores = np.empty(T, np.float64)
    _lib().or_prefill_scores(_ptr(scores), _ptr(k), _ptr(v), T, Hkv, d)
    return scores


def prefill_select(scores, cu, budget):
    """Keep set per prompt: the `budget` highest-ranking tokens in prompt order
    (ties evict the earlier token; NaN ranks as -inf).  scores [T] (any float
    dtype, widened to fp64), cu [B+1].  Returns (keep_idx [B, budget] int32,
    -1 after the last kept token; kept_len [B] int32)."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    cu = _c(cu, np.int32)
    B = cu.size - 1
    keep = np.empty((B, budget), np.int32)
    kept = np.empty(B, np.int32)
    _lib().or_prefill_select(_ptr(keep), _ptr(kept), _ptr(scores), _ptr(cu), B, budget)
    return keep, kept


def prefill_pack(k, v, cu, keep_idx, kept_len, k_cache, v_cache, block_stride, bt, bs):
    """Write the kept prompt rows at positions 0.. of each sequence through the
    block table (pools flat uint16, modified in place)."""
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    cu = _c(cu, np.int32)
    keep_idx = _c(keep_idx, np.int32)
    kept_len = _c(kept_len, np.int32)
    bt = _c(bt, np.int32)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    assert k_cache.dtype == np.uint16 and v_cache.dtype == np.uint16
    T, Hkv, d = k.shape
    B, MB = bt.shape
    _lib().or_prefill_pack(_ptr(k), _ptr(v), _ptr(cu), _ptr(keep_idx), _ptr(kept_len),
                           keep_idx.shape[1], _ptr(k_cache), _ptr(v_cache), block_stride,
                           _ptr(bt), MB, B, Hkv, d, bs)


def evict_compact(bt, ctx_lens, evict, bs):
    """Remove the evicted logical block from each table.  Returns new copies
    (bt [B, MB] int32, ctx_lens [B] int32, freed [B] int32)."""
    bt = np.array(bt, dtype=np.int32, order="C", copy=True)
    ctx = np.array(ctx_lens, dtype=np.int32, copy=True)
    evict = _c(evict, np.int32)
    B, MB = bt.shape
    freed = np.empty(B, np.int32)
    _lib().or_evict_compact(_ptr(bt), _ptr(ctx), _ptr(freed), _ptr(evict), B, MB, bs)
    return bt, ctx, freed


def select_evict_threshold(scores, ctx_lens, bs, used_blocks, total_blocks, eviction_ratio,
                           importance_threshold):
    """Threshold policy: once used_blocks > (1 - eviction_ratio) * total_blocks,
    every full block with mean importance below importance_threshold is marked,
    else the lowest-mean full block.  Returns (mask [B, MB] uint8, count [B] int32,
    means [B, MB] float64)."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    ctx_lens = _c(ctx_lens, np.int32)
    B, T, Hkv = scores.shape
    MB = T // bs
    mask = np.empty((B, MB), np.uint8)
    count = np.empty(B, np.int32)
    means = np.empty((B, MB), np.float64)
    _lib().or_select_evict_threshold(_ptr(mask), _ptr(count), _ptr(means), _ptr(scores),
                                     _ptr(ctx_lens), B, MB, Hkv, bs, int(used_blocks),
                                     int(total_blocks), float(eviction_ratio),
                                     float(importance_threshold))
    return mask, count, means


def evict_compact_mask(bt, ctx_lens, mask, bs):
    """Remove every marked full block.  Returns new copies (bt, ctx_lens, freed
    [B, MB] int32 listing freed ids in logical order, -1 after the last)."""
    bt = np.array(bt, dtype=np.int32, order="C", copy=True)
    ctx = np.array(ctx_lens, dtype=np.int32, copy=True)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    B, MB = bt.shape
    freed = np.empty((B, MB), np.int32)
    _lib().or_evict_compact_mask(_ptr(bt), _ptr(ctx), _ptr(freed), _ptr(mask), B, MB, bs)
    return bt, ctx, freed


# --------------------------------------------------------------------------- chunked prefill
def paged_prefill(q, cu_q, k_cache, v_cache, block_stride, bt, ctx_lens, Hkv, bs, scale):
    """fp64 multi-query paged attention: the q_len_b query tokens of sequence b
    are its last q_len_b cached tokens and attend causally.  q [Tq, Hq, d] bf16
    bits, cu_q [B+1] int32.  Returns out [Tq, Hq, d] float64."""
    q = _c(q, np.uint16)
    cu_q = _c(cu_q, np.int32)
    k_cache = _c(k_cache, np.uint16)
    v_cache = _c(v_cache, np.uint16)
    bt = _c(bt, np.int32)
    ctx_lens = _c(ctx_lens, np.int32)
    Tq, Hq, d = q.shape
    B, MB = bt.shape
    out = np.empty((Tq, Hq, d), np.float64)
    _lib().or_paged_prefill(_ptr(out), _ptr(q), _ptr(cu_q), _ptr(k_cache), _ptr(v_cache),
                            block_stride, _ptr(bt), MB, _ptr(ctx_lens), B, Hq, Hkv, d, bs, scale)
    return out
