"""Parity at the benchmark's full sizes, in the launch configuration bench.py times
(its Runner, automatic partitioning), on sampled sequences the oracle computes one
by one, plus properties checked on every output (finite, equal to the unsplit
decode).  The oracle reads host copies of the generator's inputs taken before the
GPU step runs."""
import numpy as np
import pytest
import torch

import bench
from helpers import (assert_attention_close, assert_evict_consistent, assert_scores_close,
                     oracle_step)
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu

SAMPLES = {
    # workload: (layers checked, sequences checked)
    "c3": ((0, 31), (0, 17, 63)),
    "c4": ((0,), (2,)),
    "c5": ((0,), (0, 64, 127)),
    "c2": ((0, 15), (0, 9, 31)),
}


@pytest.fixture(autouse=True)
def _free():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("key", list(SAMPLES))
def test_full_size_sampled(key):
    cfg = W.CONFIGS[key]
    layers, seqs = SAMPLES[key]
    dev = torch.device("cuda")
    wl = W.generate(cfg, dev)
    refs = {l: oracle_step(wl, l, seqs) for l in layers}
    evict_ref = None
    if cfg.score:  # eviction decisions of every sequence of the last layer
        evict_ref = oracle_step(wl, layers[-1], range(cfg.batch), score=True)
    r = bench.Runner(cfg, dev, wl=wl)
    r.step()
    torch.cuda.synchronize()
    assert r.err.item() == 0
    assert torch.isfinite(r.out.float()).all()
    for l in layers:
        assert_attention_close(r.out[l, list(seqs)], refs[l]["out"], f"{key} layer {l}")
    if evict_ref is not None:
        l = layers[-1]
        B, MB = r.bt.shape
        scores = torch.zeros(B, MB * cfg.block_size, cfg.hkv, dtype=torch.float32, device=dev)
        evict = torch.empty(B, dtype=torch.int32, device=dev)
        pk.pe_score_tokens(scores, wl.k_pool[l], wl.v_pool[l], r.bt, r.ctx, r.err)
        pk.pe_select_evict_block(evict, scores, r.ctx, cfg.block_size)
        torch.cuda.synchronize()
        got = scores.cpu().numpy()
        for b in range(B):
            n = int(wl.ctx_lens[b])
            assert_scores_close(got[b, :n], evict_ref["scores"][b, :n], f"seq {b}")
        n_exact = assert_evict_consistent(evict.cpu().numpy(), evict_ref["evict"],
                                          evict_ref["means"], evict_ref["gap"], key)
        assert n_exact >= B - 2


def test_full_size_128k_split_equals_unsplit():
    """Every output of the 128K workload: the automatic split-KV decode agrees with a
    single-partition decode (a property that holds at any size)."""
    cfg = W.CONFIGS["c4"]
    dev = torch.device("cuda")
    wl = W.generate(cfg, dev)
    r = bench.Runner(cfg, dev, wl=wl)
    r.step()
    split = r.out[0].clone()
    one = torch.empty_like(split)
    ws1 = pk.alloc_workspace(cfg.batch, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block_size,
                             wl.max_blocks, 1, dev)
    pk.pa_decode(one, r.q[0], wl.k_pool[0], wl.v_pool[0], r.bt, r.ctx, wl.scale, r.err, ws1, 1)
    torch.cuda.synchronize()
    assert r.err.item() == 0
    a = split.float().cpu().numpy().astype(np.float64)
    b = one.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(a - b) <= 2 * (2e-3 + 1e-2 * np.abs(b)))
