"""Incremental PagedEviction scoring on the GPU: the scored append writes each
token's ||V||/||K|| into a paged score pool; the pooled block selection reads it
through the block table.  Checked against the fp64 oracle (scores 1e-5
relative; decisions exact where the oracle's margin allows, else consistent)
and, on given fp32 scores, bit-exactly against the oracle's fp64 block means."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_evict_consistent, assert_scores_close, oracle_step
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _history(wl, layer):
    """Each sequence's cached tokens in order, gathered from the generator's pool
    (data movement only): list of [1, old_len, Hkv, d] bf16 tensors."""
    out = []
    bs = wl.cfg.block_size
    for b in range(wl.cfg.batch):
        n = int(wl.old_lens[b])
        ids = torch.as_tensor(wl.block_tables[b, :-(-n // bs)].astype(np.int64))
        k = wl.k_pool[layer].index_select(0, ids).reshape(-1, wl.cfg.hkv, wl.cfg.head_dim)[:n]
        v = wl.v_pool[layer].index_select(0, ids).reshape(-1, wl.cfg.hkv, wl.cfg.head_dim)[:n]
        out.append((k.unsqueeze(0).contiguous(), v.unsqueeze(0).contiguous()))
    return out


@pytest.mark.parametrize("key,d,bs", [("c2", 64, 16), ("c3", 128, 16), ("c2", 64, 1),
                                      ("c3", 128, 5)])
def test_scored_append_and_pooled_select(key, d, bs):
    cfg = W.scaled(W.CONFIGS[key], key="sc", layers=1, batch=6, head_dim=d, block_size=bs,
                   old_lens=(40, 15, 16, 300, 1, 129), old_len_range=(), outlier_frac=0.0)
    wl = W.generate(cfg, "cpu")
    dev = "cuda"
    N, bs, Hkv = wl.num_blocks, cfg.block_size, cfg.hkv
    bt = torch.as_tensor(wl.block_tables, device=dev)
    kc = torch.zeros(N, bs, Hkv, d, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    kc_plain, vc_plain = torch.zeros_like(kc), torch.zeros_like(vc)
    pool = torch.full((N, bs, Hkv), float("nan"), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    zero = torch.zeros(1, dtype=torch.int32, device=dev)
    for b, (k, v) in enumerate(_history(wl, 0)):     # prompt-style scored appends
        pk.pa_append_kv_scored(k.to(dev), v.to(dev), kc, vc, pool, bt[b:b + 1], zero, err)
        pk.pa_append_kv(k.to(dev), v.to(dev), kc_plain, vc_plain, bt[b:b + 1], zero, err)
    pos = torch.as_tensor(wl.positions, device=dev)   # the decode step's new token
    pk.pa_append_kv_scored(wl.k_new[0].to(dev), wl.v_new[0].to(dev), kc, vc, pool, bt, pos, err)
    pk.pa_append_kv(wl.k_new[0].to(dev), wl.v_new[0].to(dev), kc_plain, vc_plain, bt, pos, err)
    evict = torch.empty(cfg.batch, dtype=torch.int32, device=dev)
    means = torch.empty(cfg.batch, wl.max_blocks, dtype=torch.float32, device=dev)
    ctx = torch.as_tensor(wl.ctx_lens, device=dev)
    pk.pe_select_evict_block_pooled(evict, pool, bt, ctx, err, means)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert torch.equal(kc, kc_plain) and torch.equal(vc, vc_plain)  # same K/V as the plain append
    # oracle on the generator's inputs
    s = W.compact(wl, 0, range(cfg.batch))
    kco, vco = s["k_pool"].ravel().copy(), s["v_pool"].ravel().copy()
    stride = bs * Hkv * d
    oracle.append_kv(s["k_new"], s["v_new"], kco, vco, stride, s["block_tables"], s["positions"],
                     bs)
    sc = oracle.score_tokens(kco, vco, stride, s["block_tables"], s["ctx_lens"], Hkv, d, bs)
    ev, om, gap = oracle.select_evict_block(sc, s["ctx_lens"], bs)
    got_pool = pool.cpu().numpy()
    for b in range(cfg.batch):
        n = int(wl.ctx_lens[b])
        ids = wl.block_tables[b, :-(-n // bs)]
        got = got_pool[ids].reshape(-1, Hkv)[:n]
        assert_scores_close(got, sc[b, :n], f"seq {b}")
    assert_evict_consistent(evict.cpu().numpy(), ev, om, gap, key)


def test_pooled_select_is_bit_exact_on_given_scores():
    rng = np.random.default_rng(21)
    B, MB, bs, Hkv, N = 7, 9, 16, 8, 80
    perm = rng.permutation(N).astype(np.int32)
    bt = perm[:B * MB].reshape(B, MB).copy()
    pool = rng.uniform(0.5, 2.0, (N, bs, Hkv)).astype(np.float32)
    lens = np.array([0, 15, 16, 33, 144, 100, 70], np.int32)
    pool[bt[4, 5]] = 0.3                      # planted lowest block (logical 5) of sequence 4
    logical = pool[bt].reshape(B, MB * bs, Hkv)  # scores in logical order (test-side gather)
    ev, om, _ = oracle.select_evict_block(logical, lens, bs)
    dev = "cuda"
    evict = torch.empty(B, dtype=torch.int32, device=dev)
    means = torch.empty(B, MB, dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pk.pe_select_evict_block_pooled(evict, torch.as_tensor(pool).to(dev),
                                    torch.as_tensor(bt).to(dev), torch.as_tensor(lens).to(dev),
                                    err, means)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert evict.cpu().numpy().tolist() == ev.tolist() and ev[4] == 5 and ev[0] == -1
    gm = means.cpu().numpy()
    ok = ~np.isnan(om)
    assert np.array_equal(np.isnan(gm), ~ok) and np.array_equal(gm[ok], om[ok].astype(np.float32))


def test_int8_scored_append_scores_dequantised_rows():
    cfg = W.scaled(W.CONFIGS["c5"], key="i8sc", batch=3, old_lens=(50, 16, 200))
    wl = W.generate(cfg, "cpu")
    dev = "cuda"
    N, bs, Hkv, d = wl.num_blocks, cfg.block_size, cfg.hkv, cfg.head_dim
    bt = torch.as_tensor(wl.block_tables, device=dev)
    kq = torch.zeros(N, bs, Hkv, d, dtype=torch.int8, device=dev)
    vq = torch.zeros_like(kq)
    ks = torch.zeros(N, bs, Hkv, dtype=torch.float32, device=dev)
    vs = torch.zeros_like(ks)
    pool = torch.zeros_like(ks)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    zero = torch.zeros(1, dtype=torch.int32, device=dev)
    for b in range(cfg.batch):
        n = int(wl.old_lens[b])
        pk.pa_append_kv_int8_scored(wl.k_hist[0, b:b + 1, :n].contiguous().to(dev),
                                    wl.v_hist[0, b:b + 1, :n].contiguous().to(dev), kq, vq, ks, vs,
                                    pool, bt[b:b + 1], zero, err)
    pos = torch.as_tensor(wl.positions, device=dev)
    pk.pa_append_kv_int8_scored(wl.k_new[0].to(dev), wl.v_new[0].to(dev), kq, vq, ks, vs, pool,
                                bt, pos, err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ids = torch.as_tensor(wl.block_tables[wl.block_tables >= 0].astype(np.int64), device=dev)
    # the oracle quantises the generator's history itself (its own append)
    ref_step = oracle_step(wl, 0, range(cfg.batch))
    s = ref_step["compact"]
    n_blk = s["num_blocks"]
    ref = oracle.score_tokens_int8(ref_step["kq"], ref_step["vq"], ref_step["ks"], ref_step["vs"],
                                   bs * Hkv * d, s["block_tables"], s["ctx_lens"], Hkv, d, bs)
    got = pool[ids].cpu().numpy().reshape(n_blk * bs, Hkv)
    for b in range(cfg.batch):
        n = int(wl.ctx_lens[b])
        rows = np.concatenate([np.arange(j * bs, (j + 1) * bs)
                               for j in s["block_tables"][b, :-(-n // bs)]])[:n]
        assert_scores_close(got[rows], ref[b, :n], f"seq {b}")
