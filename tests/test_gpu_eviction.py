"""GPU parity of the threshold eviction policy and of the multi-block table
compaction, through the C ABI, against the fp64 oracle.

Masks, counts, tables, lengths and freed ids bit-exact; where a decision rests
on GPU block means of fp32 scores, it must match the oracle's wherever the
oracle's margin exceeds what fp32 scores can move a mean by."""
import numpy as np
import pytest
import torch

import oracle
from helpers import SCORE_RTOL, assert_attention_close
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _run_threshold(scores, lens, bs, used, total, ratio, thr):
    B, T, Hkv = scores.shape
    MB = T // bs
    mask = torch.full((B, MB), 7, dtype=torch.uint8, device="cuda")
    count = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    means = torch.empty(B, MB, dtype=torch.float32, device="cuda")
    pk.pe_select_evict_threshold(mask, count, torch.as_tensor(scores, dtype=torch.float32).cuda(),
                                 torch.as_tensor(lens).cuda(), bs, used, total, ratio, thr,
                                 block_means=means)
    torch.cuda.synchronize()
    return mask.cpu().numpy(), count.cpu().numpy(), means.cpu().numpy()


@pytest.mark.parametrize("used,total", [(80, 100), (81, 100), (1000, 1000), (0, 0)])
def test_threshold_policy_dyadic_means_bit_exact(used, total):
    """Block-constant dyadic scores: every mean is exact on both sides, so the
    masks must agree exactly, on both sides of the trigger."""
    bs, Hkv = 16, 8
    consts = [[0.5, 0.0625, 2.0, 0.09375, 0.125, 3.0, 0.1171875],
              [1.0, 2.0, 4.0, 0.5, 0.25, 8.0, 16.0],       # none below: the argmin (0.25)
              [0.03125, 0.03125, 1.0, 1.0, 1.0, 1.0, 1.0],  # two equal low blocks
              [1.0] * 7]
    tails = [5, 0, 15, 0]
    lens = []
    MB = 8
    s = np.full((len(consts), MB * bs, Hkv), 0.0, np.float32)
    for b, (c, t) in enumerate(zip(consts, tails)):
        for j, v in enumerate(c):
            s[b, j * bs:(j + 1) * bs] = v
        s[b, 7 * bs:7 * bs + t] = 0.001
        lens.append(7 * bs + t)
    lens = np.array(lens + [3], np.int32)         # plus a sequence with no full block
    s = np.concatenate([s, np.full((1, MB * bs, Hkv), 0.001, np.float32)])
    ref_mask, ref_count, ref_means = oracle.select_evict_threshold(s, lens, bs, used, total, 0.2,
                                                                   0.125)
    mask, count, means = _run_threshold(s, lens, bs, used, total, 0.2, 0.125)
    assert np.array_equal(mask, ref_mask)
    assert np.array_equal(count, ref_count)
    ok = ~np.isnan(ref_means)
    assert np.array_equal(np.isnan(means), ~ok)
    assert np.array_equal(means[ok], ref_means[ok].astype(np.float32))


def test_threshold_policy_random_scores_with_margins():
    rng = np.random.default_rng(31)
    B, MB, bs, Hkv = 48, 40, 16, 8
    lens = rng.integers(0, MB * bs + 1, B).astype(np.int32)
    # positive scores around the threshold, block-correlated so whole blocks dip
    level = rng.uniform(0.05, 0.6, (B, MB, 1, 1))
    s = (level * rng.uniform(0.5, 1.5, (B, MB, bs, Hkv))).reshape(B, MB * bs, Hkv)
    s = s.astype(np.float32)
    thr = 0.25
    ref_mask, ref_count, ref_means = oracle.select_evict_threshold(s, lens, bs, 95, 100, 0.2, thr)
    mask, count, means = _run_threshold(s, lens, bs, 95, 100, 0.2, thr)
    _, _, gap = oracle.select_evict_block(s, lens, bs)
    n_checked = 0
    for b in range(B):
        m = ref_means[b]
        cand = ~np.isnan(m)
        if (np.abs(m[cand] - thr) <= 4 * SCORE_RTOL * thr).any():
            continue        # a block mean within fp32 reach of the threshold
        if cand.any() and not (m[cand] < thr).any() and \
                gap[b] <= 4 * SCORE_RTOL * np.abs(m[cand]).min():
            continue        # the argmin fallback is a near-tie
        assert np.array_equal(mask[b], ref_mask[b]), b
        assert count[b] == ref_count[b], b
        n_checked += 1
    assert n_checked >= B - 2


def _tables(lens, bs, MB, seed):
    rng = np.random.default_rng(seed)
    N = int(sum(-(-int(n) // bs) for n in lens)) + 5
    perm = rng.permutation(N).astype(np.int32)
    bt = np.full((len(lens), MB), -1, np.int32)
    c = 0
    for b, n in enumerate(lens):
        m = -(-int(n) // bs)
        bt[b, :m] = perm[c:c + m]
        c += m
    return bt


@pytest.mark.parametrize("bs", [16, 256, 1, 5])
def test_compact_mask_bit_exact(bs):
    rng = np.random.default_rng(40 + bs)
    B, MB = 40, 100
    lens = rng.integers(0, MB * bs + 1, B).astype(np.int32)
    lens[:3] = [0, MB * bs, bs]
    bt = _tables(lens, bs, MB, seed=bs)
    nfull = lens // bs
    mask = np.zeros((B, MB), np.uint8)
    for b in range(B):
        if nfull[b]:
            k = rng.integers(0, min(nfull[b], 70) + 1)
            mask[b, rng.choice(nfull[b], size=k, replace=False)] = 1
    mask[1, :] = 1                  # a full table losing every block
    ref_bt, ref_len, ref_fr = oracle.evict_compact_mask(bt, lens, mask, bs)
    bt_d = torch.as_tensor(bt).cuda()
    len_d = torch.as_tensor(lens).cuda()
    freed = torch.full((B, MB), -9, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.pe_evict_compact_mask(bt_d, len_d, torch.as_tensor(mask).cuda(), bs, err, freed)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert np.array_equal(bt_d.cpu().numpy(), ref_bt)
    assert np.array_equal(len_d.cpu().numpy(), ref_len)
    assert np.array_equal(freed.cpu().numpy(), ref_fr)


def test_compact_mask_flags_partial_block_marks():
    bs = 16
    lens = np.array([40, 33], np.int32)               # blocks: 2 full + partial each
    bt = np.array([[3, 8, 1], [0, 5, 2]], np.int32)
    mask = np.array([[0, 1, 1], [1, 0, 0]], np.uint8)  # seq 0 marks its partial block
    ref_bt, ref_len, ref_fr = oracle.evict_compact_mask(bt, lens, mask, bs)
    bt_d = torch.as_tensor(bt).cuda()
    len_d = torch.as_tensor(lens).cuda()
    freed = torch.empty(2, 3, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.pe_evict_compact_mask(bt_d, len_d, torch.as_tensor(mask).cuda(), bs, err, freed)
    torch.cuda.synchronize()
    assert err.item() == pk.PA_DEV_BAD_EVICT
    assert np.array_equal(bt_d.cpu().numpy(), ref_bt)
    assert np.array_equal(len_d.cpu().numpy(), ref_len)
    assert np.array_equal(freed.cpu().numpy(), ref_fr)
    assert ref_bt.tolist() == [[3, 1, -1], [5, 2, -1]] and ref_len.tolist() == [24, 17]


def test_threshold_round_trip_then_decode():
    """Scores, threshold policy and compaction on the device, then a decode
    over the compacted tables: equal to the oracle doing the same from its own
    scores (low-importance blocks planted by scaling V by 0.05)."""
    cfg = W.scaled(W.CONFIGS["c2"], key="thr-rt", layers=1, batch=5,
                   old_lens=(1024, 300, 47, 15, 513))
    wl = W.generate(cfg, "cpu")
    B, MB, bs, Hkv, d = cfg.batch, wl.max_blocks, cfg.block_size, cfg.hkv, cfg.head_dim
    # plant: logical blocks 3 and 10 of sequence 0 and block 1 of sequence 2
    for b, j in [(0, 3), (0, 10), (2, 1)]:
        wl.v_pool[0, int(wl.block_tables[b, j])] *= 0.05
    kp, vp = wl.k_pool[0].cuda(), wl.v_pool[0].cuda()
    bt_d = torch.as_tensor(wl.block_tables).cuda()
    ctx = torch.as_tensor(wl.old_lens).cuda()
    scores = torch.empty(B, MB * bs, Hkv, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.pe_score_tokens(scores, kp, vp, bt_d, ctx, err)
    mask = torch.empty(B, MB, dtype=torch.uint8, device="cuda")
    count = torch.empty(B, dtype=torch.int32, device="cuda")
    pk.pe_select_evict_threshold(mask, count, scores, ctx, bs, 90, 100, 0.2, 0.1)
    freed = torch.empty(B, MB, dtype=torch.int32, device="cuda")
    pk.pe_evict_compact_mask(bt_d, ctx, mask, bs, err, freed)
    out = torch.empty(B, cfg.hq, d, dtype=torch.bfloat16, device="cuda")
    ws = pk.alloc_workspace(B, cfg.hq, Hkv, d, bs, MB, 0, "cuda")
    pk.pa_decode(out, wl.q[0].cuda(), kp, vp, bt_d, ctx, wl.scale, err, ws)
    torch.cuda.synchronize()
    assert err.item() == 0
    s = W.compact(wl, 0, range(B))
    stride = bs * Hkv * d
    kc, vc = s["k_pool"].ravel(), s["v_pool"].ravel()
    sc = oracle.score_tokens(kc, vc, stride, s["block_tables"], s["old_lens"], Hkv, d, bs)
    ref_mask, ref_count, _ = oracle.select_evict_threshold(sc, s["old_lens"], bs, 90, 100, 0.2,
                                                           0.1)
    assert np.array_equal(mask.cpu().numpy(), ref_mask)
    assert ref_mask[0, 3] and ref_mask[0, 10] and ref_mask[2, 1]
    bt_c, len_c, _ = oracle.evict_compact_mask(s["block_tables"], s["old_lens"], ref_mask, bs)
    assert np.array_equal(ctx.cpu().numpy(), len_c)
    ref = oracle.paged_decode(s["q"], kc, vc, stride, bt_c, len_c, Hkv, bs, wl.scale)
    assert_attention_close(out, ref, "decode after threshold eviction")
