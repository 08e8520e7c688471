"""pa_decode_static_scratch: decode for callers that cannot allocate device memory.

Such a caller (a runtime that owns all GPU memory, a plain-C host holding only
the pointers it was given, a process that reserved its budget at start-up)
gets its scratch from a fixed array inside the library instead of a workspace.
These tests call it through the C ABI and check its output against the fp64
oracle, element by element within the attention tolerance the parity tests
use, and against pa_decode on the same inputs: on two calls in a row, after a
call that left NaN partials in the array, and when the automatic partition
count needs more scratch than the array holds.  The file sorts last so that a
failure here stops a -x run only after every other test has run."""
import pytest
import torch

from helpers import assert_attention_close, oracle_step
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu

STATIC_BYTES = 16 * 1024 * 1024


def _inputs(cfg):
    """Device copies of one layer of a workload that appends nothing (the decode attends
    the cached tokens as they are, on both sides)."""
    assert not cfg.append
    wl = W.generate(cfg, "cpu")
    dev = torch.device("cuda")
    return dict(
        q=wl.q[0].to(dev), k=wl.k_pool[0].to(dev), v=wl.v_pool[0].to(dev),
        bt=torch.as_tensor(wl.block_tables, device=dev),
        ctx=torch.as_tensor(wl.ctx_lens, device=dev), scale=wl.scale, cfg=cfg, wl=wl)


def _pa_decode(x, num_splits=0):
    cfg, wl = x["cfg"], x["wl"]
    out = torch.empty_like(x["q"])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = pk.alloc_workspace(cfg.batch, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block_size,
                            wl.max_blocks, num_splits, "cuda")
    pk.pa_decode(out, x["q"], x["k"], x["v"], x["bt"], x["ctx"], x["scale"], err, ws,
                 num_splits)
    torch.cuda.synchronize()
    assert err.item() == 0
    return out


def _static(x, num_splits=0):
    out = torch.full_like(x["q"], float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.pa_decode_static_scratch(out, x["q"], x["k"], x["v"], x["bt"], x["ctx"], x["scale"], err,
                                num_splits)
    torch.cuda.synchronize()
    assert err.item() == 0
    return out


def _oracle(x):
    return oracle_step(x["wl"], 0, range(x["cfg"].batch))["out"]


def _partials(x):
    """Partial results (sequence, partition, kv-head share) the automatic plan of pa_decode
    writes for these inputs, from the plan it leaves in its workspace."""
    cfg, wl = x["cfg"], x["wl"]
    ws = pk.alloc_workspace(cfg.batch, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block_size,
                            wl.max_blocks, 0, "cuda")
    out = torch.empty_like(x["q"])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.pa_decode(out, x["q"], x["k"], x["v"], x["bt"], x["ctx"], x["scale"], err, ws)
    torch.cuda.synchronize()
    _, _, ns = pk.workspace_plan(ws, cfg.batch)
    return sum(ns) * max(1, 8 // cfg.hkv)


def test_static_scratch_decode_matches_the_oracle_on_two_calls():
    # call 1: several partitions per sequence (partials live in the static array);
    # call 2: other sizes, so stale contents of call 1 would show up if read.  Both
    # plans fit the array, so each call launches what pa_decode launches.
    a = _inputs(W.scaled(W.CONFIGS["c3"], key="sa", layers=1, batch=6,
                         old_len_range=(1, 3000), outlier_frac=0.0, append=False))
    b = _inputs(W.scaled(W.CONFIGS["c4"], key="sb", batch=2, old_lens=(2048, 700)))
    for x, name in ((a, "first call"), (b, "second call")):
        got = _static(x)
        assert_attention_close(got, _oracle(x), name)
        assert torch.equal(got, _pa_decode(x)), name


def test_static_scratch_never_reads_stale_partials():
    """A first call over a V pool full of NaN leaves NaN partial results in the array; a
    second call of another shape whose plan writes more partials than the first must
    still match the oracle (it reads only what it wrote)."""
    a = _inputs(W.scaled(W.CONFIGS["c3"], key="nan1", layers=1, batch=3,
                         old_lens=(900, 400, 2000), outlier_frac=0.0, append=False))
    a["v"].fill_(float("nan"))
    b = _inputs(W.scaled(W.CONFIGS["c3"], key="nan2", layers=1, batch=9,
                         old_len_range=(1500, 6000), outlier_frac=0.0, append=False))
    assert _partials(b) > _partials(a) > a["cfg"].batch
    got_a = _static(a)
    assert torch.isnan(got_a.float()).all()      # NaN values in, NaN partials and output
    got_b = _static(b)
    assert_attention_close(got_b, _oracle(b), "call after NaN partials")
    assert torch.equal(_static(b), got_b)       # and again, bit for bit


def test_static_scratch_shrinks_the_partition_count_to_fit():
    """4 sequences of 65536 tokens (block 256): the automatic plan's scratch is more than
    the array holds, so num_splits = 0 takes the largest partition count that fits."""
    cfg = W.scaled(W.CONFIGS["c4"], key="fit", batch=4, old_lens=(65536,) * 4)
    x = _inputs(cfg)
    wl = x["wl"]
    args = (cfg.batch, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block_size, wl.max_blocks)
    assert pk.pa_decode_workspace_bytes(*args, 0) > STATIC_BYTES
    auto_s = pk.pa_decode_plan(*args, 0)[0]
    fit = max(s for s in range(1, auto_s + 1)
              if pk.pa_decode_workspace_bytes(*args, s) <= STATIC_BYTES)
    assert fit < auto_s
    got = _static(x)
    assert_attention_close(got, _oracle(x), "shrunk partition count")
    # the same explicit count through pa_decode launches the same kernels
    assert torch.equal(got, _pa_decode(x, num_splits=fit))


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
