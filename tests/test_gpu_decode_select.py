"""GPU: decode and pooled block selection in one call (pa_decode_select_pooled,
pa_decode_planned_select_pooled) against the two separate calls and the fp64 oracle.

The selection runs in extra CTAs at the front of the decode's merge launch (or, where
the decode has no warp-per-row merge, as its own kernel after it).  Either way the
attention output must be bit for bit pa_decode's, the evicted block and the block
means bit for bit pe_select_evict_block_pooled's, and the evicted block the oracle's
on the same fp32 scores ([KVL] "PagedEviction 块级驱逐机制": the lowest mean among the
complete blocks, ties to the lowest index)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import Device, assert_attention_close, oracle_step
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu

C = W.CONFIGS
CASES = {
    # c2 at its batch: balanced split, warp-per-row merge carrying the selection CTAs
    "c2": (W.scaled(C["c2"], key="ds2", layers=1, score=False), 0),
    # two long sequences: one CTA per merged row, the selection as its own kernel
    "few-long": (W.scaled(C["c3"], key="dsfl", layers=1, batch=2, old_lens=(6000, 3000),
                          outlier_frac=0.0), 0),
    # one partition per sequence: no merge launch, the selection as its own kernel
    "direct": (W.scaled(C["c3"], key="dsd", layers=1, batch=5,
                        old_lens=(300, 17, 16, 1000, 64), outlier_frac=0.0), 1),
    # block size 12: the general-shape kernel
    "general": (W.scaled(C["c3"], key="dsg", layers=1, batch=4, block_size=12,
                         old_lens=(100, 37, 12, 300), outlier_frac=0.0), 0),
    # one-token and three-token blocks: every cached token a block, or nearly
    "bs1": (W.scaled(C["c3"], key="ds1", layers=1, batch=3, block_size=1,
                     old_lens=(50, 1, 7), outlier_frac=0.0), 0),
    "bs3": (W.scaled(C["c3"], key="ds3", layers=1, batch=4, block_size=3,
                     old_lens=(100, 2, 3, 301), outlier_frac=0.0), 0),
}


def _score_pool(wl, seed):
    """Random fp32 scores [N, bs, Hkv] with a planted lowest block in sequence 0."""
    rng = np.random.default_rng(seed)
    cfg = wl.cfg
    pool = rng.uniform(0.5, 2.0, (wl.num_blocks, cfg.block_size, cfg.hkv)).astype(np.float32)
    n_full = int(wl.ctx_lens[0]) // cfg.block_size
    if n_full > 1:
        pool[wl.block_tables[0, n_full - 1]] = 0.25
    return pool


def _oracle_select(wl, pool):
    bs, MB = wl.cfg.block_size, wl.max_blocks
    bt = np.where(wl.block_tables >= 0, wl.block_tables, 0)
    logical = pool[bt].reshape(wl.cfg.batch, MB * bs, wl.cfg.hkv)   # test-side gather
    ev, om, _ = oracle.select_evict_block(logical, np.asarray(wl.ctx_lens, np.int32), bs)
    return ev, om


@pytest.mark.parametrize("planned", [False, True])
@pytest.mark.parametrize("key", list(CASES))
def test_decode_with_selection_equals_the_two_calls(key, planned):
    cfg, splits = CASES[key]
    wl = W.generate(cfg, "cpu")
    ref = oracle_step(wl, 0, range(cfg.batch))
    dev = Device(wl, num_splits=splits)
    dev.step(0)                        # append, then the plain decode
    torch.cuda.synchronize()
    assert dev.err.item() == 0
    out_ref = dev.out[0].clone()
    assert_attention_close(out_ref, ref["out"], key)
    pool_np = _score_pool(wl, 7)
    pool = torch.as_tensor(pool_np).cuda()
    B, MB = wl.cfg.batch, wl.max_blocks
    ev_ref = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    mean_ref = torch.empty(B, MB, dtype=torch.float32, device="cuda")
    pk.pe_select_evict_block_pooled(ev_ref, pool, dev.bt, dev.ctx, dev.err, mean_ref)
    out = torch.full_like(out_ref, float("nan"))
    ev = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    means = torch.full((B, MB), 7.0, dtype=torch.float32, device="cuda")
    args = (out, dev.q[0], dev.k_pool[0], dev.v_pool[0], dev.bt, dev.ctx, wl.scale, dev.err, ev,
            pool, means, dev.ws, splits)
    if planned:
        pk.pa_decode_prepare(dev.q[0], dev.k_pool[0], dev.bt, dev.ctx, dev.err, dev.ws, splits)
        for _ in range(2):             # the kept plan serves repeated calls
            pk.pa_decode_planned_select_pooled(*args)
    else:
        pk.pa_decode_select_pooled(*args)
    torch.cuda.synchronize()
    assert dev.err.item() == 0
    assert torch.equal(out, out_ref), key
    assert torch.equal(ev, ev_ref), key
    assert np.array_equal(means.cpu().numpy(), mean_ref.cpu().numpy(), equal_nan=True)
    oev, om = _oracle_select(wl, pool_np)
    assert ev.cpu().numpy().tolist() == oev.tolist()
    gm = means.cpu().numpy()
    ok = ~np.isnan(om)
    assert np.array_equal(np.isnan(gm), ~ok) and np.array_equal(gm[ok], om[ok].astype(np.float32))


def test_selection_without_block_means():
    cfg, splits = CASES["c2"]
    wl = W.generate(cfg, "cpu")
    dev = Device(wl)
    dev.step(0)
    pool = torch.as_tensor(_score_pool(wl, 3)).cuda()
    ev = torch.full((cfg.batch,), -9, dtype=torch.int32, device="cuda")
    out = torch.empty_like(dev.out[0])
    pk.pa_decode_select_pooled(out, dev.q[0], dev.k_pool[0], dev.v_pool[0], dev.bt, dev.ctx,
                               wl.scale, dev.err, ev, pool, None, dev.ws)
    torch.cuda.synchronize()
    assert dev.err.item() == 0
    assert torch.equal(out, dev.out[0])
    oev, _ = _oracle_select(wl, pool.cpu().numpy())
    assert ev.cpu().numpy().tolist() == oev.tolist()
