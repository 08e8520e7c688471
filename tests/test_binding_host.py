"""CPU test of the Python binding's marshalling and argument checks.

The library is replaced by a recorder and the CUDA-residency check by a dtype
check, so the binding runs on CPU tensors: valid calls reach the C entry point
with the sizes, strides and pointers the tensors imply; tensors too short for
the batch, a missing error flag, mismatched inner dims or a tensor on another
device are refused before any call."""
import pytest
import torch

from paged_kv_cache_396_b200 import pagedkv as pk


class _Recorder:
    def __init__(self):
        self.calls = []

    def pa_status_string(self, code):
        return b"recorded"

    def __getattr__(self, name):
        def entry(*args):
            self.calls.append((name, args))
            return 0
        return entry


class _Stream:
    cuda_stream = 0


@pytest.fixture
def lib(monkeypatch):
    rec = _Recorder()
    monkeypatch.setattr(pk, "load", lambda *a, **k: rec)

    def want_dtype(t, dtype, name):
        if t.dtype != dtype:
            raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    monkeypatch.setattr(pk, "_want", want_dtype)
    return rec


B, HQ, HKV, D, BS, N, MB = 3, 8, 2, 64, 16, 12, 4
ST = _Stream()


def _i32(*shape, fill=0):
    return torch.full(shape, fill, dtype=torch.int32)


def _decode_args(pad=0):
    big = torch.zeros(N, BS + pad, HKV, D, dtype=torch.bfloat16)
    pool = big[:, :BS]
    return dict(out=torch.empty(B, HQ, D, dtype=torch.bfloat16),
                q=torch.zeros(B, HQ, D, dtype=torch.bfloat16), k_cache=pool, v_cache=pool,
                block_tables=_i32(B, MB), ctx_lens=_i32(B, fill=5), scale=0.125,
                err_flag=_i32(1))


def test_decode_marshals_sizes_and_the_block_stride(lib):
    a = _decode_args(pad=3)
    pk.pa_decode(**a, stream=ST)
    name, args = lib.calls[-1]
    assert name == "pa_decode"
    assert args[4] == (BS + 3) * HKV * D                  # block stride from stride(0)
    assert args[6] == MB and args[8:14] == (B, HQ, HKV, D, BS, N)
    assert args[0].value == a["out"].data_ptr() and args[2].value == a["k_cache"].data_ptr()


@pytest.mark.parametrize("bad", ["ctx_short", "table_rows", "err_empty", "pool_dtype",
                                 "other_device", "q_shape"])
def test_decode_refuses_before_calling(lib, bad):
    a = _decode_args()
    if bad == "ctx_short":
        a["ctx_lens"] = _i32(B - 1)
    elif bad == "table_rows":
        a["block_tables"] = _i32(B - 1, MB)
    elif bad == "err_empty":
        a["err_flag"] = _i32(0)
    elif bad == "pool_dtype":
        a["k_cache"] = a["v_cache"] = torch.zeros(N, BS, HKV, D, dtype=torch.float16)
    elif bad == "other_device":
        a["ctx_lens"] = torch.empty(B, dtype=torch.int32, device="meta")
    elif bad == "q_shape":
        a["q"] = torch.zeros(B, HQ, D + 1, dtype=torch.bfloat16)
    with pytest.raises((ValueError, TypeError)):
        pk.pa_decode(**a, stream=ST)
    assert lib.calls == []


def test_longer_index_arrays_are_accepted(lib):
    """The kernels read the first B entries, so longer arrays are valid input."""
    a = _decode_args()
    a["ctx_lens"] = _i32(B + 4, fill=5)
    a["block_tables"] = _i32(B + 2, MB)
    pk.pa_decode(**a, stream=ST)
    assert lib.calls[-1][0] == "pa_decode"


def _append_args(kind="bf16", n_new=2):
    dt = {"bf16": torch.bfloat16, "int8": torch.int8, "fp8": torch.uint8}[kind]
    pool = torch.zeros(N, BS, HKV, D, dtype=dt)
    a = dict(k_new=torch.zeros(B, n_new, HKV, D, dtype=torch.bfloat16),
             v_new=torch.zeros(B, n_new, HKV, D, dtype=torch.bfloat16))
    if kind == "int8":
        sc = torch.zeros(N, BS, HKV)
        a.update(kq_cache=pool, vq_cache=pool, k_scale=sc, v_scale=sc)
    elif kind == "fp8":
        a.update(k8_cache=pool, v8_cache=pool)
    else:
        a.update(k_cache=pool, v_cache=pool)
    a.update(block_tables=_i32(B, MB), positions=_i32(B), err_flag=_i32(1),
             slot_out=torch.empty(B, n_new, dtype=torch.int64))
    return a


APPENDS = {"bf16": "pa_append_kv", "int8": "pa_append_kv_int8", "fp8": "pa_append_kv_fp8"}


@pytest.mark.parametrize("kind", list(APPENDS))
def test_appends_marshal_and_refuse(lib, kind):
    fn = getattr(pk, APPENDS[kind])
    fn(**_append_args(kind), stream=ST)
    assert lib.calls[-1][0] == APPENDS[kind]
    lib.calls.clear()
    for change in ("positions", "slot_out", "inner", "rows"):
        a = _append_args(kind)
        if change == "positions":
            a["positions"] = _i32(B - 1)
        elif change == "slot_out":
            a["slot_out"] = torch.empty(B, dtype=torch.int64)        # B*n_new needed
        elif change == "inner":
            a["k_new"] = a["v_new"] = torch.zeros(B, 2, HKV, D // 2, dtype=torch.bfloat16)
        else:
            a["block_tables"] = _i32(B - 2, MB)
        with pytest.raises(ValueError):
            fn(**a, stream=ST)
    assert lib.calls == []


def test_eviction_calls_refuse_short_outputs(lib):
    scores = torch.zeros(B, MB * BS, HKV)
    with pytest.raises(ValueError):
        pk.pe_select_evict_block(_i32(B - 1), scores, _i32(B), BS, stream=ST)
    with pytest.raises(ValueError):
        pk.pe_select_evict_threshold(torch.zeros(B, MB, dtype=torch.uint8), _i32(B - 1), scores,
                                     _i32(B), BS, 90, 100, stream=ST)
    with pytest.raises(ValueError):
        pk.pe_select_evict_threshold(torch.zeros(B, MB, dtype=torch.uint8), _i32(B), scores,
                                     _i32(B), BS, 90, 100, block_means=torch.zeros(B, MB + 1),
                                     stream=ST)
    with pytest.raises(ValueError):
        pk.pe_evict_compact(_i32(B, MB), _i32(B), _i32(B - 1), BS, _i32(1), stream=ST)
    with pytest.raises(ValueError):
        pk.pe_evict_compact_mask(_i32(B, MB), _i32(B - 1), torch.zeros(B, MB, dtype=torch.uint8),
                                 BS, _i32(1), stream=ST)
    assert lib.calls == []
    pk.pe_select_evict_block(_i32(B), scores, _i32(B), BS, stream=ST)
    pk.pe_evict_compact(_i32(B, MB), _i32(B), _i32(B), BS, _i32(1), stream=ST)
    assert [c[0] for c in lib.calls] == ["pe_select_evict_block", "pe_evict_compact"]


def test_prefill_attention_refuses_short_lengths(lib):
    a = _decode_args()
    cu = torch.tensor([0, 2, 3, 5], dtype=torch.int32)
    q = torch.zeros(5, HQ, D, dtype=torch.bfloat16)
    out = torch.empty_like(q)
    with pytest.raises(ValueError):
        pk.pa_prefill_attention(out, q, cu, 2, a["k_cache"], a["v_cache"], a["block_tables"],
                                _i32(B - 1), 0.125, a["err_flag"], stream=ST)
    assert lib.calls == []
    pk.pa_prefill_attention(out, q, cu, 2, a["k_cache"], a["v_cache"], a["block_tables"],
                            a["ctx_lens"], 0.125, a["err_flag"], stream=ST)
    assert lib.calls[-1][0] == "pa_prefill_attention"
