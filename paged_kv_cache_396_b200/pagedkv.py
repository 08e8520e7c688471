"""Thin Python binding of libpagedkv.so (the C ABI in include/pagedkv.h).

Argument marshalling only: every function takes torch CUDA tensors, checks
dtypes and layouts, reads sizes from shapes and strides, and calls the C entry
point of the same name on the current (or given) CUDA stream.  All the work runs
in the library's kernels; there is no CPU fallback, and a missing library is an
error.

Tensor conventions (the C header has the full statement of each operation):
  pools      [N, bs, Hkv, d] (bf16 or int8); the block stride is stride(0), so a
             view into a larger tensor such as the nano-vLLM [2, L, N, bs, Hkv, d]
             works unchanged.  Inner three dims must be contiguous.
  scales     [N, bs, Hkv] float32, contiguous (INT8 pools).
  block_tables [B, MB] int32, ctx_lens/positions [B] int32, err_flag [>=1] int32.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")

PA_OK = 0
PA_DEV_BAD_BLOCK = 1
PA_DEV_BAD_LEN = 2
PA_DEV_TIMEOUT = 4
PA_DEV_BAD_EVICT = 8
PA_DEV_BAD_PLAN = 16

EXPORTED = (
    "pa_status_string", "pa_version", "pa_append_kv", "pa_decode_workspace_bytes", "pa_decode_plan",
    "pa_decode",
    "pe_score_tokens", "pe_select_evict_block", "pa_append_kv_int8", "pa_decode_int8",
    "pa_decode_static_scratch", "pa_decode_prepare", "pa_decode_planned",
    "pa_decode_int8_planned", "pa_decode_fp8_planned", "pa_decode_select_pooled",
    "pa_decode_planned_select_pooled", "pa_append_kv_scored",
    "pa_append_kv_int8_scored",
    "pe_select_evict_block_pooled", "pa_append_kv_fp8", "pa_decode_fp8",
    "pe_prefill_scores", "pe_prefill_select", "pe_prefill_pack", "pe_prefill_compress",
    "pe_evict_compact", "pe_select_evict_threshold", "pe_evict_compact_mask",
    "pa_prefill_attention", "pa_prefill_attention_workspace_bytes", "pa_selftest_wait_timeout",
)


class PagedKVError(RuntimeError):
    def __init__(self, fn: str, code: int, text: str):
        super().__init__(f"{fn} failed with status {code}: {text}")
        self.code = code


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the shared library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libpagedkv.so not found at {path}; build it with "
                          "`python -m paged_kv_cache_396_b200.build_lib`")
    lib = ctypes.CDLL(path)
    p, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                            ctypes.c_size_t)
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_status_string.argtypes = [i32]
    lib.pa_version.restype = ctypes.c_char_p
    lib.pa_version.argtypes = []
    lib.pa_append_kv.restype = i32
    lib.pa_append_kv.argtypes = [p, p, p, p, i64, p, i32, p, i32, i32, i32, i32, i32, i64, p, p, p]
    lib.pa_append_kv_int8.restype = i32
    lib.pa_append_kv_int8.argtypes = [p, p, p, p, p, p, i64, p, i32, p, i32, i32, i32, i32, i32,
                                      i64, p, p, p]
    lib.pa_decode_workspace_bytes.restype = sz
    lib.pa_decode_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32]
    lib.pa_decode_plan.restype = i32
    lib.pa_decode_plan.argtypes = [i32, i32, i32, i32, i32, i32, i32, p, p, p, p]
    lib.pa_decode.restype = i32
    lib.pa_decode.argtypes = [p, p, p, p, i64, p, i32, p, i32, i32, i32, i32, i32, i64, f32, i32,
                              p, sz, p, p]
    lib.pa_decode_int8.restype = i32
    lib.pa_decode_int8.argtypes = [p, p, p, p, p, p, i64, p, i32, p, i32, i32, i32, i32, i32, i64,
                                   f32, i32, p, sz, p, p]
    lib.pa_decode_prepare.restype = i32
    lib.pa_decode_prepare.argtypes = [p, i32, i32, i32, i32, i32, i32, i32, p, sz, p, p]
    lib.pa_decode_planned.restype = i32
    lib.pa_decode_planned.argtypes = lib.pa_decode.argtypes
    # pa_decode's arguments with (evict, block_means, score_pool) before err_flag
    sel_args = lib.pa_decode.argtypes[:-2] + [p, p, p] + lib.pa_decode.argtypes[-2:]
    lib.pa_decode_select_pooled.restype = i32
    lib.pa_decode_select_pooled.argtypes = sel_args
    lib.pa_decode_planned_select_pooled.restype = i32
    lib.pa_decode_planned_select_pooled.argtypes = sel_args
    lib.pa_decode_int8_planned.restype = i32
    lib.pa_decode_int8_planned.argtypes = lib.pa_decode_int8.argtypes
    lib.pa_decode_static_scratch.restype = i32
    lib.pa_decode_static_scratch.argtypes = [p, p, p, p, i64, p, i32, p, i32, i32, i32, i32, i32,
                                             i64, f32, i32, p, p]
    lib.pa_append_kv_scored.restype = i32
    lib.pa_append_kv_scored.argtypes = [p, p, p, p, i64, p, p, i32, p, i32, i32, i32, i32, i32,
                                        i64, p, p, p]
    lib.pa_append_kv_int8_scored.restype = i32
    lib.pa_append_kv_int8_scored.argtypes = [p, p, p, p, p, p, p, i64, p, i32, p, i32, i32, i32,
                                             i32, i32, i64, p, p, p]
    lib.pe_select_evict_block_pooled.restype = i32
    lib.pe_select_evict_block_pooled.argtypes = [p, p, p, p, i32, p, i32, i32, i32, i64, p, p]
    lib.pa_append_kv_fp8.restype = i32
    lib.pa_append_kv_fp8.argtypes = [p, p, p, p, i64, p, i32, p, i32, i32, i32, i32, i32, i64, p,
                                     p, p]
    lib.pa_decode_fp8.restype = i32
    lib.pa_decode_fp8.argtypes = [p, p, p, p, i64, p, i32, p, i32, i32, i32, i32, i32, i64, f32,
                                  i32, p, sz, p, p]
    lib.pa_decode_fp8_planned.restype = i32
    lib.pa_decode_fp8_planned.argtypes = lib.pa_decode_fp8.argtypes
    lib.pe_prefill_scores.restype = i32
    lib.pe_prefill_scores.argtypes = [p, p, p, i64, i32, i32, p]
    lib.pe_prefill_select.restype = i32
    lib.pe_prefill_select.argtypes = [p, p, p, p, i32, i32, p, p]
    lib.pe_prefill_pack.restype = i32
    lib.pe_prefill_pack.argtypes = [p, p, i64, p, i32, p, p, p, p, p, i32, i32, i32, i32, i32,
                                    i64, p, p]
    lib.pe_prefill_compress.restype = i32
    lib.pe_prefill_compress.argtypes = [p, p, i64, p, i32, p, p, p, i64, i32, i32, i32, i32, i32,
                                        i64, p, p, p, p, p]
    lib.pe_evict_compact.restype = i32
    lib.pe_evict_compact.argtypes = [p, i32, p, p, p, i32, i32, p, p]
    lib.pe_select_evict_threshold.restype = i32
    lib.pe_select_evict_threshold.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i64, i64,
                                              ctypes.c_double, ctypes.c_double, p]
    lib.pe_evict_compact_mask.restype = i32
    lib.pe_evict_compact_mask.argtypes = [p, i32, p, p, p, i32, i32, p, p]
    lib.pa_prefill_attention.restype = i32
    lib.pa_prefill_attention.argtypes = [p, p, p, i32, p, p, i64, p, i32, p, i32, i32, i32, i32,
                                         i32, i64, f32, p, p, sz, p]
    lib.pa_prefill_attention_workspace_bytes.restype = sz
    lib.pa_selftest_wait_timeout.restype = i32
    lib.pa_selftest_wait_timeout.argtypes = [p, p]
    lib.pa_prefill_attention_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
    lib.pe_score_tokens.restype = i32
    lib.pe_score_tokens.argtypes = [p, p, p, i64, p, i32, p, i32, i32, i32, i32, i64, p, p]
    lib.pe_select_evict_block.restype = i32
    lib.pe_select_evict_block.argtypes = [p, p, p, p, i32, i32, i32, i32, p]
    _lib = lib
    return lib


def _check(fn: str, code: int):
    if code != PA_OK:
        raise PagedKVError(fn, code, load().pa_status_string(code).decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _want(t: torch.Tensor, dtype, name: str):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise TypeError(f"{name}: expected a CUDA tensor")


def _covers(t: torch.Tensor, n: int, name: str):
    """t holds at least the n elements the kernels read (they index by batch row)."""
    if t.numel() < n:
        raise ValueError(f"{name}: needs at least {n} elements, got {t.numel()}")


def _table_rows(block_tables: torch.Tensor, B: int):
    if block_tables.dim() != 2 or block_tables.shape[0] < B or block_tables.shape[1] < 1:
        raise ValueError(f"block_tables: expected [B >= {B}, MB >= 1], got "
                         f"{tuple(block_tables.shape)}")


def _one_device(ref: torch.Tensor, *ts):
    """Every tensor the call reads or writes is on the pools' device."""
    for t in ts:
        if t is not None and t.device != ref.device:
            raise ValueError(f"all tensors must be on {ref.device}, got one on {t.device}")


def _pool_geometry(pool: torch.Tensor, name: str):
    if pool.dim() != 4:
        raise ValueError(f"{name}: expected [N, bs, Hkv, d], got shape {tuple(pool.shape)}")
    N, bs, Hkv, d = pool.shape
    if pool.stride(3) != 1 or pool.stride(2) != d or pool.stride(1) != Hkv * d:
        raise ValueError(f"{name}: the [bs, Hkv, d] part must be contiguous")
    return N, bs, Hkv, d, pool.stride(0)


def _same_pool(a: torch.Tensor, b: torch.Tensor):
    if a.shape != b.shape or a.stride() != b.stride():
        raise ValueError("K and V pools must have the same shape and strides")


# ----------------------------------------------------------------------------- append
def _append_sizes(k_new, Hkv, d, block_tables, positions, err_flag, slot_out, B, n_new):
    if tuple(k_new.shape[2:]) != (Hkv, d):
        raise ValueError("k_new inner dims must match the pool's [Hkv, d]")
    _table_rows(block_tables, B)
    _covers(positions, B, "positions")
    _covers(err_flag, 1, "err_flag")
    if slot_out is not None:
        _want(slot_out, torch.int64, "slot_out")
        _covers(slot_out, B * n_new, "slot_out")


def pa_append_kv(k_new, v_new, k_cache, v_cache, block_tables, positions, err_flag,
                 slot_out=None, stream=None):
    """Write new tokens into the paged pools.  k_new/v_new: [B, n_new, Hkv, d] or
    [B, Hkv, d] bf16 (contiguous); positions [B]: position of each sequence's
    first new token.  slot_out: optional [B, n_new] int64."""
    for t, n in ((k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _want(t, torch.bfloat16, n)
    _want(block_tables, torch.int32, "block_tables")
    _want(positions, torch.int32, "positions")
    _want(err_flag, torch.int32, "err_flag")
    N, bs, Hkv, d, stride = _pool_geometry(k_cache, "k_cache")
    _same_pool(k_cache, v_cache)
    if k_new.dim() == 3:
        k_new, v_new = k_new.unsqueeze(1), v_new.unsqueeze(1)
    if not (k_new.is_contiguous() and v_new.is_contiguous()) or k_new.shape != v_new.shape:
        raise ValueError("k_new/v_new must be contiguous and of equal shape")
    B, n_new = k_new.shape[0], k_new.shape[1]
    _append_sizes(k_new, Hkv, d, block_tables, positions, err_flag, slot_out, B, n_new)
    _one_device(k_cache, k_new, v_new, block_tables, positions, err_flag, slot_out)
    bt = block_tables.contiguous()
    rc = load().pa_append_kv(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), stride,
                             _ptr(bt), bt.shape[1], _ptr(positions.contiguous()), B, n_new, Hkv, d,
                             bs, N, _ptr(slot_out), _ptr(err_flag), _stream(stream))
    _check("pa_append_kv", rc)


def pa_append_kv_int8(k_new, v_new, kq_cache, vq_cache, k_scale, v_scale, block_tables,
                      positions, err_flag, slot_out=None, stream=None):
    """Quantise (symmetric INT8, one fp32 scale per (token, kv head)) and write
    new tokens.  Pools [N, bs, Hkv, d] int8, scales [N, bs, Hkv] float32."""
    _want(k_new, torch.bfloat16, "k_new")
    _want(v_new, torch.bfloat16, "v_new")
    _want(kq_cache, torch.int8, "kq_cache")
    _want(vq_cache, torch.int8, "vq_cache")
    _want(k_scale, torch.float32, "k_scale")
    _want(v_scale, torch.float32, "v_scale")
    _want(block_tables, torch.int32, "block_tables")
    _want(positions, torch.int32, "positions")
    _want(err_flag, torch.int32, "err_flag")
    N, bs, Hkv, d, stride = _pool_geometry(kq_cache, "kq_cache")
    _same_pool(kq_cache, vq_cache)
    for s in (k_scale, v_scale):
        if tuple(s.shape) != (N, bs, Hkv) or not s.is_contiguous():
            raise ValueError("scale pools must be contiguous [N, bs, Hkv]")
    if k_new.dim() == 3:
        k_new, v_new = k_new.unsqueeze(1), v_new.unsqueeze(1)
    if not (k_new.is_contiguous() and v_new.is_contiguous()) or k_new.shape != v_new.shape:
        raise ValueError("k_new/v_new must be contiguous and of equal shape")
    B, n_new = k_new.shape[0], k_new.shape[1]
    _append_sizes(k_new, Hkv, d, block_tables, positions, err_flag, slot_out, B, n_new)
    _one_device(kq_cache, k_new, v_new, k_scale, v_scale, block_tables, positions, err_flag,
                slot_out)
    bt = block_tables.contiguous()
    rc = load().pa_append_kv_int8(_ptr(k_new), _ptr(v_new), _ptr(kq_cache), _ptr(vq_cache),
                                  _ptr(k_scale), _ptr(v_scale), stride, _ptr(bt), bt.shape[1],
                                  _ptr(positions.contiguous()), B, n_new, Hkv, d, bs, N,
                                  _ptr(slot_out), _ptr(err_flag), _stream(stream))
    _check("pa_append_kv_int8", rc)


# ----------------------------------------------------------------------------- decode
def pa_decode_workspace_bytes(B, Hq, Hkv, d, bs, max_blocks_per_seq, num_splits=0) -> int:
    return int(load().pa_decode_workspace_bytes(B, Hq, Hkv, d, bs, max_blocks_per_seq,
                                                num_splits))


def pa_decode_plan(B, Hq, Hkv, d, bs, max_blocks_per_seq, num_splits=0):
    """(partitions per sequence at most, tokens per partition, kernel launches per
    call, staged tensor-core kernel or not) that pa_decode will use for these sizes."""
    s, c, n, k = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check("pa_decode_plan", load().pa_decode_plan(B, Hq, Hkv, d, bs, max_blocks_per_seq,
                                                   num_splits, ctypes.byref(s), ctypes.byref(c),
                                                   ctypes.byref(n), ctypes.byref(k)))
    return s.value, c.value, n.value, bool(k.value)


def workspace_plan(workspace, B):
    """Diagnostic: the partition plan the staged decode kernel left in its
    workspace on the last call (header: unit counter, unit count, partition
    tokens; then partitions per sequence at byte 256).  Returns
    (n_units, chunk_tokens, partitions_per_sequence[B]) on the host."""
    head = workspace[:16].view(torch.int32).cpu().tolist()
    ns = workspace[256:256 + 4 * B].view(torch.int32).cpu().tolist()
    return head[1], head[2], ns


def alloc_workspace(B, Hq, Hkv, d, bs, max_blocks_per_seq, num_splits=0, device=None):
    """Convenience: a device byte tensor of the size pa_decode needs (or None)."""
    n = pa_decode_workspace_bytes(B, Hq, Hkv, d, bs, max_blocks_per_seq, num_splits)
    return torch.zeros(n, dtype=torch.uint8, device=device) if n else None


def _decode_checks(out, q, block_tables, ctx_lens, err_flag):
    _want(out, torch.bfloat16, "out")
    _want(q, torch.bfloat16, "q")
    _want(block_tables, torch.int32, "block_tables")
    _want(ctx_lens, torch.int32, "ctx_lens")
    _want(err_flag, torch.int32, "err_flag")
    if not (out.is_contiguous() and q.is_contiguous()) or out.shape != q.shape or q.dim() != 3:
        raise ValueError("q and out must be contiguous [B, Hq, d] of equal shape")
    B = q.shape[0]
    _table_rows(block_tables, B)
    _covers(ctx_lens, B, "ctx_lens")
    _covers(err_flag, 1, "err_flag")


def pa_decode(out, q, k_cache, v_cache, block_tables, ctx_lens, scale, err_flag,
              workspace=None, num_splits=0, stream=None):
    """Paged decode attention (bf16 pools): out[b, i] = softmax(scale q.K) V over
    the ctx_lens[b] tokens of sequence b, kv head i // (Hq/Hkv)."""
    _decode_bf16("pa_decode", out, q, k_cache, v_cache, block_tables, ctx_lens, scale, err_flag,
                 workspace, num_splits, stream)


def pa_decode_planned(out, q, k_cache, v_cache, block_tables, ctx_lens, scale, err_flag,
                      workspace=None, num_splits=0, stream=None):
    """pa_decode with the partition plan pa_decode_prepare left in the workspace."""
    _decode_bf16("pa_decode_planned", out, q, k_cache, v_cache, block_tables, ctx_lens, scale,
                 err_flag, workspace, num_splits, stream)


def pa_decode_prepare(q, k_cache, block_tables, ctx_lens, err_flag, workspace, num_splits=0,
                      stream=None):
    """Write the partition plan of ctx_lens into the workspace for the planned decode
    calls of the same sizes (q [B, Hq, d] and the pool [N, bs, Hkv, d], bf16 or one-byte,
    give the sizes)."""
    _want(block_tables, torch.int32, "block_tables")
    _want(ctx_lens, torch.int32, "ctx_lens")
    _want(err_flag, torch.int32, "err_flag")
    N, bs, Hkv, d, _ = _pool_geometry(k_cache, "k_cache")
    if q.dim() != 3 or q.shape[2] != d:
        raise ValueError("q must be [B, Hq, d] with the pool's d")
    B, Hq = q.shape[0], q.shape[1]
    _table_rows(block_tables, B)
    _covers(ctx_lens, B, "ctx_lens")
    _covers(err_flag, 1, "err_flag")
    _one_device(k_cache, block_tables, ctx_lens, err_flag, workspace)
    ws_ptr, ws_n = (None, 0) if workspace is None else (_ptr(workspace), workspace.numel() *
                                                        workspace.element_size())
    rc = load().pa_decode_prepare(_ptr(ctx_lens.contiguous()), B, Hq, Hkv, d, bs,
                                  block_tables.shape[1], int(num_splits), ws_ptr, ws_n,
                                  _ptr(err_flag), _stream(stream))
    _check("pa_decode_prepare", rc)


def _decode_bf16(fn, out, q, k_cache, v_cache, block_tables, ctx_lens, scale, err_flag,
                 workspace, num_splits, stream):
    _decode_checks(out, q, block_tables, ctx_lens, err_flag)
    _want(k_cache, torch.bfloat16, "k_cache")
    _want(v_cache, torch.bfloat16, "v_cache")
    N, bs, Hkv, d, stride = _pool_geometry(k_cache, "k_cache")
    _same_pool(k_cache, v_cache)
    B, Hq, dq = q.shape
    if dq != d:
        raise ValueError("q head_dim differs from the pool's")
    _one_device(k_cache, out, q, v_cache, block_tables, ctx_lens, err_flag, workspace)
    bt = block_tables.contiguous()
    ws_ptr, ws_n = (None, 0) if workspace is None else (_ptr(workspace), workspace.numel() *
                                                        workspace.element_size())
    rc = getattr(load(), fn)(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), stride, _ptr(bt),
                             bt.shape[1], _ptr(ctx_lens.contiguous()), B, Hq, Hkv, d, bs, N,
                             float(scale), int(num_splits), ws_ptr, ws_n, _ptr(err_flag),
                             _stream(stream))
    _check(fn, rc)


def _select_checks(evict, score_pool, block_tables, block_means):
    _want(evict, torch.int32, "evict")
    _want(score_pool, torch.float32, "score_pool")
    if score_pool.dim() != 3 or not score_pool.is_contiguous():
        raise ValueError("score_pool must be contiguous [N, bs, Hkv]")
    B, MB = block_tables.shape
    if block_means is not None:
        _want(block_means, torch.float32, "block_means")
        if tuple(block_means.shape) != (B, MB) or not block_means.is_contiguous():
            raise ValueError("block_means must be contiguous [B, MB]")
    _covers(evict, B, "evict")


def _decode_select(fn, out, q, k_cache, v_cache, block_tables, ctx_lens, scale, err_flag,
                   evict, score_pool, block_means, workspace, num_splits, stream):
    _decode_checks(out, q, block_tables, ctx_lens, err_flag)
    _want(k_cache, torch.bfloat16, "k_cache")
    _want(v_cache, torch.bfloat16, "v_cache")
    N, bs, Hkv, d, stride = _pool_geometry(k_cache, "k_cache")
    _same_pool(k_cache, v_cache)
    _select_checks(evict, score_pool, block_tables, block_means)
    if tuple(score_pool.shape) != (N, bs, Hkv):
        raise ValueError("score_pool must be [N, bs, Hkv] of the KV pool")
    B, Hq, dq = q.shape
    if dq != d:
        raise ValueError("q head_dim differs from the pool's")
    _one_device(k_cache, out, q, v_cache, block_tables, ctx_lens, err_flag, workspace, evict,
                score_pool, block_means)
    bt = block_tables.contiguous()
    ws_ptr, ws_n = (None, 0) if workspace is None else (_ptr(workspace), workspace.numel() *
                                                        workspace.element_size())
    rc = getattr(load(), fn)(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), stride, _ptr(bt),
                             bt.shape[1], _ptr(ctx_lens.contiguous()), B, Hq, Hkv, d, bs, N,
                             float(scale), int(num_splits), ws_ptr, ws_n, _ptr(evict),
                             _ptr(block_means), _ptr(score_pool), _ptr(err_flag), _stream(stream))
    _check(fn, rc)


def pa_decode_select_pooled(out, q, k_cache, v_cache, block_tables, ctx_lens, scale, err_flag,
                            evict, score_pool, block_means=None, workspace=None, num_splits=0,
                            stream=None):
    """pa_decode and pe_select_evict_block_pooled in one call: the selection runs in
    extra CTAs of the decode's merge launch, beside the decode kernel."""
    _decode_select("pa_decode_select_pooled", out, q, k_cache, v_cache, block_tables, ctx_lens,
                   scale, err_flag, evict, score_pool, block_means, workspace, num_splits, stream)


def pa_decode_planned_select_pooled(out, q, k_cache, v_cache, block_tables, ctx_lens, scale,
                                    err_flag, evict, score_pool, block_means=None, workspace=None,
                                    num_splits=0, stream=None):
    """pa_decode_select_pooled with the partition plan pa_decode_prepare left in the
    workspace."""
    _decode_select("pa_decode_planned_select_pooled", out, q, k_cache, v_cache, block_tables,
                   ctx_lens, scale, err_flag, evict, score_pool, block_means, workspace,
                   num_splits, stream)


def pa_decode_static_scratch(out, q, k_cache, v_cache, block_tables, ctx_lens, scale, err_flag,
                             num_splits=0, stream=None):
    """pa_decode for callers that cannot allocate device memory: the same result,
    with scratch taken from a fixed 16 MiB array inside the library (shared by all
    calls on a device; calls that overlap on the GPU race).  num_splits=0 picks the
    largest partition count that fits; sizes that cannot fit raise PagedKVError."""
    _decode_checks(out, q, block_tables, ctx_lens, err_flag)
    _want(k_cache, torch.bfloat16, "k_cache")
    _want(v_cache, torch.bfloat16, "v_cache")
    N, bs, Hkv, d, stride = _pool_geometry(k_cache, "k_cache")
    _same_pool(k_cache, v_cache)
    B, Hq, dq = q.shape
    if dq != d:
        raise ValueError("q head_dim differs from the pool's")
    _one_device(k_cache, out, q, v_cache, block_tables, ctx_lens, err_flag)
    bt = block_tables.contiguous()
    rc = load().pa_decode_static_scratch(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), stride,
                                         _ptr(bt), bt.shape[1], _ptr(ctx_lens.contiguous()), B, Hq,
                                         Hkv, d, bs, N, float(scale), int(num_splits),
                                         _ptr(err_flag), _stream(stream))
    _check("pa_decode_static_scratch", rc)


def pa_decode_int8(out, q, kq_cache, vq_cache, k_scale, v_scale, block_tables, ctx_lens, scale,
                   err_flag, workspace=None, num_splits=0, stream=None):
    """Paged decode attention over INT8 pools dequantised in registers."""
    _decode_int8("pa_decode_int8", out, q, kq_cache, vq_cache, k_scale, v_scale, block_tables,
                 ctx_lens, scale, err_flag, workspace, num_splits, stream)


def pa_decode_int8_planned(out, q, kq_cache, vq_cache, k_scale, v_scale, block_tables, ctx_lens,
                           scale, err_flag, workspace=None, num_splits=0, stream=None):
    """pa_decode_int8 with the partition plan pa_decode_prepare left in the workspace."""
    _decode_int8("pa_decode_int8_planned", out, q, kq_cache, vq_cache, k_scale, v_scale,
                 block_tables, ctx_lens, scale, err_flag, workspace, num_splits, stream)


def _decode_int8(fn, out, q, kq_cache, vq_cache, k_scale, v_scale, block_tables, ctx_lens, scale,
                 err_flag, workspace, num_splits, stream):
    _decode_checks(out, q, block_tables, ctx_lens, err_flag)
    _want(kq_cache, torch.int8, "kq_cache")
    _want(vq_cache, torch.int8, "vq_cache")
    _want(k_scale, torch.float32, "k_scale")
    _want(v_scale, torch.float32, "v_scale")
    N, bs, Hkv, d, stride = _pool_geometry(kq_cache, "kq_cache")
    _same_pool(kq_cache, vq_cache)
    for s in (k_scale, v_scale):
        if tuple(s.shape) != (N, bs, Hkv) or not s.is_contiguous():
            raise ValueError("scale pools must be contiguous [N, bs, Hkv]")
    B, Hq, dq = q.shape
    if dq != d:
        raise ValueError("q head_dim differs from the pool's")
    _one_device(kq_cache, out, q, vq_cache, k_scale, v_scale, block_tables, ctx_lens, err_flag,
                workspace)
    bt = block_tables.contiguous()
    ws_ptr, ws_n = (None, 0) if workspace is None else (_ptr(workspace), workspace.numel() *
                                                        workspace.element_size())
    rc = getattr(load(), fn)(_ptr(out), _ptr(q), _ptr(kq_cache), _ptr(vq_cache),
                             _ptr(k_scale), _ptr(v_scale), stride, _ptr(bt), bt.shape[1],
                             _ptr(ctx_lens.contiguous()), B, Hq, Hkv, d, bs, N, float(scale),
                             int(num_splits), ws_ptr, ws_n, _ptr(err_flag), _stream(stream))
    _check(fn, rc)


# ----------------------------------------------------------------------------- eviction
def pe_score_tokens(scores, k_cache, v_cache, block_tables, ctx_lens, err_flag, stream=None):
    """scores [B, MB*bs, Hkv] float32 <- ||V|| / ||K|| for t < ctx_lens[b]."""
    _want(scores, torch.float32, "scores")
    _want(k_cache, torch.bfloat16, "k_cache")
    _want(v_cache, torch.bfloat16, "v_cache")
    _want(block_tables, torch.int32, "block_tables")
    _want(ctx_lens, torch.int32, "ctx_lens")
    _want(err_flag, torch.int32, "err_flag")
    N, bs, Hkv, d, stride = _pool_geometry(k_cache, "k_cache")
    _same_pool(k_cache, v_cache)
    bt = block_tables.contiguous()
    B, MB = bt.shape
    if tuple(scores.shape) != (B, MB * bs, Hkv) or not scores.is_contiguous():
        raise ValueError("scores must be contiguous [B, MB*bs, Hkv]")
    _covers(ctx_lens, B, "ctx_lens")
    _covers(err_flag, 1, "err_flag")
    _one_device(k_cache, scores, v_cache, block_tables, ctx_lens, err_flag)
    rc = load().pe_score_tokens(_ptr(scores), _ptr(k_cache), _ptr(v_cache), stride, _ptr(bt), MB,
                                _ptr(ctx_lens.contiguous()), B, Hkv, d, bs, N, _ptr(err_flag),
                                _stream(stream))
    _check("pe_score_tokens", rc)


def pe_select_evict_block(evict, scores, ctx_lens, bs, block_means=None, stream=None):
    """evict [B] int32 <- lowest-mean full block per sequence (-1 if none)."""
    _want(evict, torch.int32, "evict")
    _want(scores, torch.float32, "scores")
    _want(ctx_lens, torch.int32, "ctx_lens")
    B, T, Hkv = scores.shape
    if T % bs:
        raise ValueError("scores' token dim must be MB*bs")
    MB = T // bs
    if block_means is not None:
        _want(block_means, torch.float32, "block_means")
        if tuple(block_means.shape) != (B, MB) or not block_means.is_contiguous():
            raise ValueError("block_means must be contiguous [B, MB]")
    _covers(evict, B, "evict")
    _covers(ctx_lens, B, "ctx_lens")
    _one_device(scores, evict, ctx_lens, block_means)
    rc = load().pe_select_evict_block(_ptr(evict), _ptr(block_means), _ptr(scores.contiguous()),
                                      _ptr(ctx_lens.contiguous()), B, MB, Hkv, bs,
                                      _stream(stream))
    _check("pe_select_evict_block", rc)


# ----------------------------------------------------------------------------- incremental scores
def _score_pool_check(score_pool, N, bs, Hkv):
    _want(score_pool, torch.float32, "score_pool")
    if tuple(score_pool.shape) != (N, bs, Hkv) or not score_pool.is_contiguous():
        raise ValueError("score_pool must be contiguous [N, bs, Hkv] float32")


def pa_append_kv_scored(k_new, v_new, k_cache, v_cache, score_pool, block_tables, positions,
                        err_flag, slot_out=None, stream=None):
    """pa_append_kv that also writes each new (token, kv head) importance
    ||V|| / ||K|| into score_pool [N, bs, Hkv] (paged like the KV pool)."""
    for t, n in ((k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _want(t, torch.bfloat16, n)
    _want(block_tables, torch.int32, "block_tables")
    _want(positions, torch.int32, "positions")
    _want(err_flag, torch.int32, "err_flag")
    N, bs, Hkv, d, stride = _pool_geometry(k_cache, "k_cache")
    _same_pool(k_cache, v_cache)
    _score_pool_check(score_pool, N, bs, Hkv)
    if k_new.dim() == 3:
        k_new, v_new = k_new.unsqueeze(1), v_new.unsqueeze(1)
    if not (k_new.is_contiguous() and v_new.is_contiguous()) or k_new.shape != v_new.shape:
        raise ValueError("k_new/v_new must be contiguous and of equal shape")
    B, n_new = k_new.shape[0], k_new.shape[1]
    _append_sizes(k_new, Hkv, d, block_tables, positions, err_flag, slot_out, B, n_new)
    _one_device(k_cache, k_new, v_new, score_pool, block_tables, positions, err_flag, slot_out)
    bt = block_tables.contiguous()
    rc = load().pa_append_kv_scored(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                    stride, _ptr(score_pool), _ptr(bt), bt.shape[1],
                                    _ptr(positions.contiguous()), B, n_new, Hkv, d, bs, N,
                                    _ptr(slot_out), _ptr(err_flag), _stream(stream))
    _check("pa_append_kv_scored", rc)


def pa_append_kv_int8_scored(k_new, v_new, kq_cache, vq_cache, k_scale, v_scale, score_pool,
                             block_tables, positions, err_flag, slot_out=None, stream=None):
    """pa_append_kv_int8 that also stores the importance of each dequantised
    new row into score_pool [N, bs, Hkv]."""
    _want(k_new, torch.bfloat16, "k_new")
    _want(v_new, torch.bfloat16, "v_new")
    _want(kq_cache, torch.int8, "kq_cache")
    _want(vq_cache, torch.int8, "vq_cache")
    _want(k_scale, torch.float32, "k_scale")
    _want(v_scale, torch.float32, "v_scale")
    _want(block_tables, torch.int32, "block_tables")
    _want(positions, torch.int32, "positions")
    _want(err_flag, torch.int32, "err_flag")
    N, bs, Hkv, d, stride = _pool_geometry(kq_cache, "kq_cache")
    _same_pool(kq_cache, vq_cache)
    for sp in (k_scale, v_scale):
        if tuple(sp.shape) != (N, bs, Hkv) or not sp.is_contiguous():
            raise ValueError("scale pools must be contiguous [N, bs, Hkv]")
    _score_pool_check(score_pool, N, bs, Hkv)
    if k_new.dim() == 3:
        k_new, v_new = k_new.unsqueeze(1), v_new.unsqueeze(1)
    if not (k_new.is_contiguous() and v_new.is_contiguous()) or k_new.shape != v_new.shape:
        raise ValueError("k_new/v_new must be contiguous and of equal shape")
    B, n_new = k_new.shape[0], k_new.shape[1]
    _append_sizes(k_new, Hkv, d, block_tables, positions, err_flag, slot_out, B, n_new)
    _one_device(kq_cache, k_new, v_new, k_scale, v_scale, score_pool, block_tables, positions,
                err_flag, slot_out)
    bt = block_tables.contiguous()
    rc = load().pa_append_kv_int8_scored(_ptr(k_new), _ptr(v_new), _ptr(kq_cache),
                                         _ptr(vq_cache), _ptr(k_scale), _ptr(v_scale),
                                         _ptr(score_pool), stride, _ptr(bt), bt.shape[1],
                                         _ptr(positions.contiguous()), B, n_new, Hkv, d, bs, N,
                                         _ptr(slot_out), _ptr(err_flag), _stream(stream))
    _check("pa_append_kv_int8_scored", rc)


def pe_select_evict_block_pooled(evict, score_pool, block_tables, ctx_lens, err_flag,
                                 block_means=None, stream=None):
    """Lowest-mean full block per sequence, scores read from score_pool
    [N, bs, Hkv] through the block table (no K/V pass)."""
    _want(evict, torch.int32, "evict")
    _want(score_pool, torch.float32, "score_pool")
    _want(block_tables, torch.int32, "block_tables")
    _want(ctx_lens, torch.int32, "ctx_lens")
    _want(err_flag, torch.int32, "err_flag")
    N, bs, Hkv = score_pool.shape
    if not score_pool.is_contiguous():
        raise ValueError("score_pool must be contiguous")
    bt = block_tables.contiguous()
    B, MB = bt.shape
    if block_means is not None:
        _want(block_means, torch.float32, "block_means")
        if tuple(block_means.shape) != (B, MB) or not block_means.is_contiguous():
            raise ValueError("block_means must be contiguous [B, MB]")
    _covers(evict, B, "evict")
    _covers(ctx_lens, B, "ctx_lens")
    _covers(err_flag, 1, "err_flag")
    _one_device(score_pool, evict, block_tables, ctx_lens, err_flag, block_means)
    rc = load().pe_select_evict_block_pooled(_ptr(evict), _ptr(block_means), _ptr(score_pool),
                                             _ptr(bt), MB, _ptr(ctx_lens.contiguous()), B, Hkv,
                                             bs, N, _ptr(err_flag), _stream(stream))
    _check("pe_select_evict_block_pooled", rc)


# ----------------------------------------------------------------------------- fp8
def pa_append_kv_fp8(k_new, v_new, k8_cache, v8_cache, block_tables, positions, err_flag,
                     slot_out=None, stream=None):
    """Cast new tokens to e4m3 (round to nearest even, saturating at 448) and
    write them.  Pools [N, bs, Hkv, d] uint8 holding e4m3 codes."""
    _want(k_new, torch.bfloat16, "k_new")
    _want(v_new, torch.bfloat16, "v_new")
    _want(k8_cache, torch.uint8, "k8_cache")
    _want(v8_cache, torch.uint8, "v8_cache")
    _want(block_tables, torch.int32, "block_tables")
    _want(positions, torch.int32, "positions")
    _want(err_flag, torch.int32, "err_flag")
    N, bs, Hkv, d, stride = _pool_geometry(k8_cache, "k8_cache")
    _same_pool(k8_cache, v8_cache)
    if k_new.dim() == 3:
        k_new, v_new = k_new.unsqueeze(1), v_new.unsqueeze(1)
    if not (k_new.is_contiguous() and v_new.is_contiguous()) or k_new.shape != v_new.shape:
        raise ValueError("k_new/v_new must be contiguous and of equal shape")
    B, n_new = k_new.shape[0], k_new.shape[1]
    _append_sizes(k_new, Hkv, d, block_tables, positions, err_flag, slot_out, B, n_new)
    _one_device(k8_cache, k_new, v_new, block_tables, positions, err_flag, slot_out)
    bt = block_tables.contiguous()
    rc = load().pa_append_kv_fp8(_ptr(k_new), _ptr(v_new), _ptr(k8_cache), _ptr(v8_cache), stride,
                                 _ptr(bt), bt.shape[1], _ptr(positions.contiguous()), B, n_new,
                                 Hkv, d, bs, N, _ptr(slot_out), _ptr(err_flag), _stream(stream))
    _check("pa_append_kv_fp8", rc)


def pa_decode_fp8(out, q, k8_cache, v8_cache, block_tables, ctx_lens, scale, err_flag,
                  workspace=None, num_splits=0, stream=None):
    """Paged decode attention over e4m3 pools, widened exactly in registers."""
    _decode_fp8("pa_decode_fp8", out, q, k8_cache, v8_cache, block_tables, ctx_lens, scale,
                err_flag, workspace, num_splits, stream)


def pa_decode_fp8_planned(out, q, k8_cache, v8_cache, block_tables, ctx_lens, scale, err_flag,
                          workspace=None, num_splits=0, stream=None):
    """pa_decode_fp8 with the partition plan pa_decode_prepare left in the workspace."""
    _decode_fp8("pa_decode_fp8_planned", out, q, k8_cache, v8_cache, block_tables, ctx_lens,
                scale, err_flag, workspace, num_splits, stream)


def _decode_fp8(fn, out, q, k8_cache, v8_cache, block_tables, ctx_lens, scale, err_flag,
                workspace, num_splits, stream):
    _decode_checks(out, q, block_tables, ctx_lens, err_flag)
    _want(k8_cache, torch.uint8, "k8_cache")
    _want(v8_cache, torch.uint8, "v8_cache")
    N, bs, Hkv, d, stride = _pool_geometry(k8_cache, "k8_cache")
    _same_pool(k8_cache, v8_cache)
    B, Hq, dq = q.shape
    if dq != d:
        raise ValueError("q head_dim differs from the pool's")
    _one_device(k8_cache, out, q, v8_cache, block_tables, ctx_lens, err_flag, workspace)
    bt = block_tables.contiguous()
    ws_ptr, ws_n = (None, 0) if workspace is None else (_ptr(workspace), workspace.numel() *
                                                        workspace.element_size())
    rc = getattr(load(), fn)(_ptr(out), _ptr(q), _ptr(k8_cache), _ptr(v8_cache), stride,
                             _ptr(bt), bt.shape[1], _ptr(ctx_lens.contiguous()), B, Hq, Hkv, d,
                             bs, N, float(scale), int(num_splits), ws_ptr, ws_n, _ptr(err_flag),
                             _stream(stream))
    _check(fn, rc)


# ----------------------------------------------------------------------------- prefill stage
def _prompt_rows(k, v):
    _want(k, torch.bfloat16, "k")
    _want(v, torch.bfloat16, "v")
    if k.dim() != 3 or k.shape != v.shape or not (k.is_contiguous() and v.is_contiguous()):
        raise ValueError("k, v: expected contiguous [T, Hkv, d] of equal shape")
    return k.shape


def pe_prefill_scores(scores, k, v, stream=None):
    """Per-token importance of concatenated prompts: head mean of ||V||/||K||.
    k, v [T, Hkv, d] bf16 contiguous; scores [T] float32."""
    T, Hkv, d = _prompt_rows(k, v)
    _want(scores, torch.float32, "scores")
    if scores.numel() < T or not scores.is_contiguous():
        raise ValueError("scores: expected a contiguous float32 tensor of T elements")
    _one_device(k, v, scores)
    _check("pe_prefill_scores", load().pe_prefill_scores(_ptr(scores), _ptr(k), _ptr(v), T, Hkv,
                                                         d, _stream(stream)))


def pe_prefill_select(keep_idx, kept_len, scores, cu_seqlens, err_flag, stream=None):
    """Indices (prompt-local, in order) of the budget highest-ranking tokens of
    each prompt.  keep_idx [B, budget] int32, kept_len [B] int32, scores [T]
    float32, cu_seqlens [B+1] int32."""
    _want(keep_idx, torch.int32, "keep_idx")
    _want(kept_len, torch.int32, "kept_len")
    _want(scores, torch.float32, "scores")
    _want(cu_seqlens, torch.int32, "cu_seqlens")
    _want(err_flag, torch.int32, "err_flag")
    B, budget = keep_idx.shape
    if not keep_idx.is_contiguous() or cu_seqlens.numel() != B + 1:
        raise ValueError("keep_idx must be contiguous [B, budget] and cu_seqlens [B+1]")
    _covers(kept_len, B, "kept_len")
    _covers(err_flag, 1, "err_flag")
    _one_device(scores, keep_idx, kept_len, cu_seqlens, err_flag)
    _check("pe_prefill_select", load().pe_prefill_select(
        _ptr(keep_idx), _ptr(kept_len), _ptr(scores), _ptr(cu_seqlens.contiguous()), B, budget,
        _ptr(err_flag), _stream(stream)))


def pe_prefill_pack(k_cache, v_cache, block_tables, k, v, cu_seqlens, keep_idx, kept_len,
                    err_flag, stream=None):
    """Write the kept prompt rows at positions 0.. of each sequence."""
    T, Hkv, d = _prompt_rows(k, v)
    _want(k_cache, torch.bfloat16, "k_cache")
    _want(v_cache, torch.bfloat16, "v_cache")
    N, bs, Hkv_c, d_c, stride = _pool_geometry(k_cache, "k_cache")
    _same_pool(k_cache, v_cache)
    if (Hkv_c, d_c) != (Hkv, d):
        raise ValueError("prompt rows and pool differ in Hkv or d")
    _want(block_tables, torch.int32, "block_tables")
    _want(cu_seqlens, torch.int32, "cu_seqlens")
    _want(keep_idx, torch.int32, "keep_idx")
    _want(kept_len, torch.int32, "kept_len")
    _want(err_flag, torch.int32, "err_flag")
    B, budget = keep_idx.shape
    if cu_seqlens.numel() != B + 1:
        raise ValueError("cu_seqlens must hold B + 1 offsets")
    _table_rows(block_tables, B)
    _covers(kept_len, B, "kept_len")
    _covers(err_flag, 1, "err_flag")
    _one_device(k_cache, v_cache, block_tables, k, v, cu_seqlens, keep_idx, kept_len, err_flag)
    bt = block_tables.contiguous()
    _check("pe_prefill_pack", load().pe_prefill_pack(
        _ptr(k_cache), _ptr(v_cache), stride, _ptr(bt), bt.shape[1], _ptr(k), _ptr(v),
        _ptr(cu_seqlens.contiguous()), _ptr(keep_idx.contiguous()), _ptr(kept_len), B, budget,
        Hkv, d, bs, N, _ptr(err_flag), _stream(stream)))


def pe_prefill_compress(k_cache, v_cache, block_tables, k, v, cu_seqlens, scores, keep_idx,
                        kept_len, err_flag, stream=None):
    """Score, select and pack in one call (budget = keep_idx.shape[1])."""
    T, Hkv, d = _prompt_rows(k, v)
    _want(k_cache, torch.bfloat16, "k_cache")
    _want(v_cache, torch.bfloat16, "v_cache")
    N, bs, Hkv_c, d_c, stride = _pool_geometry(k_cache, "k_cache")
    _same_pool(k_cache, v_cache)
    if (Hkv_c, d_c) != (Hkv, d):
        raise ValueError("prompt rows and pool differ in Hkv or d")
    _want(block_tables, torch.int32, "block_tables")
    _want(scores, torch.float32, "scores")
    _want(keep_idx, torch.int32, "keep_idx")
    _want(kept_len, torch.int32, "kept_len")
    _want(cu_seqlens, torch.int32, "cu_seqlens")
    _want(err_flag, torch.int32, "err_flag")
    B, budget = keep_idx.shape
    if scores.numel() < T or not keep_idx.is_contiguous() or cu_seqlens.numel() != B + 1:
        raise ValueError("scores [T], keep_idx contiguous [B, budget], cu_seqlens [B+1]")
    _table_rows(block_tables, B)
    _covers(kept_len, B, "kept_len")
    _covers(err_flag, 1, "err_flag")
    _one_device(k_cache, v_cache, block_tables, k, v, cu_seqlens, scores, keep_idx, kept_len,
                err_flag)
    bt = block_tables.contiguous()
    _check("pe_prefill_compress", load().pe_prefill_compress(
        _ptr(k_cache), _ptr(v_cache), stride, _ptr(bt), bt.shape[1], _ptr(k), _ptr(v),
        _ptr(cu_seqlens.contiguous()), T, B, budget, Hkv, d, bs, N, _ptr(scores),
        _ptr(keep_idx), _ptr(kept_len), _ptr(err_flag), _stream(stream)))


def pe_evict_compact(block_tables, ctx_lens, evict, block_size, err_flag, freed=None,
                     stream=None):
    """Remove each sequence's evicted logical block from its table in place
    (block_tables [B, MB] int32 contiguous, ctx_lens [B] int32 lowered by
    block_size); freed [B] int32 (optional) receives the released physical ids."""
    _want(block_tables, torch.int32, "block_tables")
    _want(ctx_lens, torch.int32, "ctx_lens")
    _want(evict, torch.int32, "evict")
    _want(err_flag, torch.int32, "err_flag")
    if not (block_tables.is_contiguous() and ctx_lens.is_contiguous()):
        raise ValueError("block_tables and ctx_lens are updated in place: pass contiguous tensors")
    if freed is not None:
        _want(freed, torch.int32, "freed")
    B, MB = block_tables.shape
    _covers(ctx_lens, B, "ctx_lens")
    _covers(evict, B, "evict")
    _covers(err_flag, 1, "err_flag")
    if freed is not None:
        _covers(freed, B, "freed")
    _one_device(block_tables, ctx_lens, evict, err_flag, freed)
    _check("pe_evict_compact", load().pe_evict_compact(
        _ptr(block_tables), MB, _ptr(ctx_lens), _ptr(freed), _ptr(evict.contiguous()), B,
        int(block_size), _ptr(err_flag), _stream(stream)))


def pe_select_evict_threshold(mask, count, scores, ctx_lens, block_size, used_blocks,
                              total_blocks, eviction_ratio=0.2, importance_threshold=0.1,
                              block_means=None, stream=None):
    """Threshold policy over token scores [B, MB*bs, Hkv]: mask [B, MB] uint8,
    count [B] int32 (block_means [B, MB] float32 optional)."""
    _want(mask, torch.uint8, "mask")
    _want(count, torch.int32, "count")
    _want(scores, torch.float32, "scores")
    _want(ctx_lens, torch.int32, "ctx_lens")
    B, T, Hkv = scores.shape
    MB = T // block_size
    if T != MB * block_size or tuple(mask.shape) != (B, MB) or not mask.is_contiguous():
        raise ValueError("scores must be [B, MB*bs, Hkv] and mask contiguous [B, MB]")
    if block_means is not None:
        _want(block_means, torch.float32, "block_means")
        if tuple(block_means.shape) != (B, MB) or not block_means.is_contiguous():
            raise ValueError("block_means must be contiguous [B, MB]")
    _covers(count, B, "count")
    _covers(ctx_lens, B, "ctx_lens")
    _one_device(scores, mask, count, ctx_lens, block_means)
    _check("pe_select_evict_threshold", load().pe_select_evict_threshold(
        _ptr(mask), _ptr(count), _ptr(block_means), _ptr(scores.contiguous()),
        _ptr(ctx_lens.contiguous()), B, MB, Hkv, int(block_size), int(used_blocks),
        int(total_blocks), float(eviction_ratio), float(importance_threshold), _stream(stream)))


def pe_evict_compact_mask(block_tables, ctx_lens, mask, block_size, err_flag, freed=None,
                          stream=None):
    """Remove every marked full block from each table in place; freed [B, MB]
    int32 (optional) lists the released physical ids, -1 padded."""
    _want(block_tables, torch.int32, "block_tables")
    _want(ctx_lens, torch.int32, "ctx_lens")
    _want(mask, torch.uint8, "mask")
    _want(err_flag, torch.int32, "err_flag")
    if not (block_tables.is_contiguous() and ctx_lens.is_contiguous()):
        raise ValueError("block_tables and ctx_lens are updated in place: pass contiguous tensors")
    B, MB = block_tables.shape
    if tuple(mask.shape) != (B, MB):
        raise ValueError("mask must be [B, MB]")
    if freed is not None:
        _want(freed, torch.int32, "freed")
        if tuple(freed.shape) != (B, MB) or not freed.is_contiguous():
            raise ValueError("freed must be contiguous [B, MB]")
    _covers(ctx_lens, B, "ctx_lens")
    _covers(err_flag, 1, "err_flag")
    _one_device(block_tables, ctx_lens, mask, err_flag, freed)
    _check("pe_evict_compact_mask", load().pe_evict_compact_mask(
        _ptr(block_tables), MB, _ptr(ctx_lens), _ptr(freed), _ptr(mask.contiguous()), B,
        int(block_size), _ptr(err_flag), _stream(stream)))


# ----------------------------------------------------------------------------- chunked prefill
def pa_prefill_attention_workspace_bytes(B, Hq, Hkv, d, bs, max_q_len) -> int:
    return int(load().pa_prefill_attention_workspace_bytes(B, Hq, Hkv, d, bs, max_q_len))


def alloc_prefill_workspace(B, Hq, Hkv, d, bs, max_q_len, device=None):
    """Convenience: a device byte tensor for pa_prefill_attention's balanced mode
    (None when that mode does not apply to these sizes)."""
    n = pa_prefill_attention_workspace_bytes(B, Hq, Hkv, d, bs, max_q_len)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def pa_prefill_attention(out, q, cu_q, max_q_len, k_cache, v_cache, block_tables, ctx_lens,
                         scale, err_flag, workspace=None, stream=None):
    """Multi-query paged attention: the q_len_b = cu_q[b+1]-cu_q[b] query rows of
    sequence b are its last q_len_b cached tokens and attend causally.
    q, out [Tq, Hq, d] bf16 contiguous; cu_q [B+1] int32; ctx_lens [B] int32.
    workspace (optional, uint8 device tensor, alloc_prefill_workspace): balances the
    work over the SMs."""
    _want(out, torch.bfloat16, "out")
    _want(q, torch.bfloat16, "q")
    _want(cu_q, torch.int32, "cu_q")
    _want(block_tables, torch.int32, "block_tables")
    _want(ctx_lens, torch.int32, "ctx_lens")
    _want(err_flag, torch.int32, "err_flag")
    _want(k_cache, torch.bfloat16, "k_cache")
    _want(v_cache, torch.bfloat16, "v_cache")
    if workspace is not None:
        _want(workspace, torch.uint8, "workspace")
    N, bs, Hkv, d, stride = _pool_geometry(k_cache, "k_cache")
    _same_pool(k_cache, v_cache)
    if q.dim() != 3 or q.shape != out.shape or not (q.is_contiguous() and out.is_contiguous()):
        raise ValueError("q and out must be contiguous [Tq, Hq, d] of equal shape")
    Tq, Hq, dq = q.shape
    if dq != d:
        raise ValueError("q head_dim differs from the pool's")
    B = block_tables.shape[0]
    if cu_q.numel() != B + 1:
        raise ValueError("cu_q must hold B + 1 offsets")
    _table_rows(block_tables, B)
    _covers(ctx_lens, B, "ctx_lens")
    _covers(err_flag, 1, "err_flag")
    _one_device(k_cache, out, q, cu_q, v_cache, block_tables, ctx_lens, err_flag, workspace)
    bt = block_tables.contiguous()
    _check("pa_prefill_attention", load().pa_prefill_attention(
        _ptr(out), _ptr(q), _ptr(cu_q.contiguous()), int(max_q_len), _ptr(k_cache),
        _ptr(v_cache), stride, _ptr(bt), bt.shape[1], _ptr(ctx_lens.contiguous()), B, Hq, Hkv, d,
        bs, N, float(scale), _ptr(err_flag), _ptr(workspace) if workspace is not None else None,
        workspace.numel() if workspace is not None else 0, _stream(stream)))


# ----------------------------------------------------------------------------- self-test
def pa_selftest_wait_timeout(err_flag, stream=None):
    """Runs the kernels' bounded wait on a phase nothing completes: after ~2 s the
    device sets PA_DEV_TIMEOUT in err_flag ([1] int32, caller-zeroed) and the kernel
    returns; the context stays usable."""
    _want(err_flag, torch.int32, "err_flag")
    _check("pa_selftest_wait_timeout",
           load().pa_selftest_wait_timeout(_ptr(err_flag), _stream(stream)))
