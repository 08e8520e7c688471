"""pa_decode_static_scratch: decode for callers that cannot allocate device memory.

Such a caller (a runtime that owns all GPU memory, a plain-C host holding only
the pointers it was given, a process that reserved its budget at start-up)
gets its scratch from a fixed array inside the library instead of a workspace.
This checks, through the C ABI, that two calls in a row give what pa_decode
gives on the same inputs, within the attention tolerance the parity tests use.
The file sorts last so that a failure here stops a -x run only after every
other test has run."""
import numpy as np
import pytest
import torch

from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2


def _inputs(cfg):
    wl = W.generate(cfg, "cpu")
    dev = torch.device("cuda")
    return dict(
        q=wl.q[0].to(dev), k=wl.k_pool[0].to(dev), v=wl.v_pool[0].to(dev),
        bt=torch.as_tensor(wl.block_tables, device=dev),
        ctx=torch.as_tensor(wl.ctx_lens, device=dev), scale=wl.scale, cfg=cfg, wl=wl)


def _reference(x):
    cfg, wl = x["cfg"], x["wl"]
    out = torch.empty_like(x["q"])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = pk.alloc_workspace(cfg.batch, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block_size,
                            wl.max_blocks, 0, "cuda")
    pk.pa_decode(out, x["q"], x["k"], x["v"], x["bt"], x["ctx"], x["scale"], err, ws)
    torch.cuda.synchronize()
    assert err.item() == 0
    return out


def _close(got, ref, what):
    g = got.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(g - r) <= ATOL + RTOL * np.abs(r)), what


def test_static_scratch_decode_matches_pa_decode_on_two_calls():
    # call 1: several partitions per sequence (partials live in the static array);
    # call 2: other sizes, so stale contents of call 1 would show up if read.
    a = _inputs(W.scaled(W.CONFIGS["c3"], key="sa", layers=1, batch=6,
                         old_len_range=(1, 3000), outlier_frac=0.0))
    b = _inputs(W.scaled(W.CONFIGS["c4"], key="sb", batch=2, old_lens=(2048, 700)))
    refs = [_reference(a), _reference(b)]
    for x, ref, name in ((a, refs[0], "first call"), (b, refs[1], "second call")):
        out = torch.full_like(x["q"], float("nan"))
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        pk.pa_decode_static_scratch(out, x["q"], x["k"], x["v"], x["bt"], x["ctx"], x["scale"],
                                    err)
        torch.cuda.synchronize()
        assert err.item() == 0
        _close(out, ref, name)


def test_static_scratch_rejects_sizes_beyond_the_array():
    # 64 sequences of up to 513 blocks of 16 tokens with 513 partitions each need
    # far more than the array holds; the call must refuse before launching.
    dev = "cuda"
    B, Hq, Hkv, d, bs, MB = 64, 32, 8, 128, 16, 513
    q = torch.zeros(B, Hq, d, dtype=torch.bfloat16, device=dev)
    pool = torch.zeros(4, bs, Hkv, d, dtype=torch.bfloat16, device=dev)
    bt = torch.zeros(B, MB, dtype=torch.int32, device=dev)
    ctx = torch.full((B,), MB * bs, dtype=torch.int32, device=dev)
    out = torch.full_like(q, 7.0)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    with pytest.raises(pk.PagedKVError) as e:
        pk.pa_decode_static_scratch(out, q, pool, pool, bt, ctx, 0.1, err, num_splits=MB)
    assert e.value.code == -4
    torch.cuda.synchronize()
    assert (out == 7.0).all() and err.item() == 0   # nothing was launched
