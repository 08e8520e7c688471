"""GPU parity of the PagedEviction prefill stage (token scores, keep set,
packing into the paged pool) and of the block-table compaction, through the C
ABI, against the fp64 oracle.

Scores within 1e-5 relative; keep sets, packed pools, tables, lengths and freed
ids bit-exact.  Where the keep decision rests on GPU-computed fp32 scores, the
oracle's decision must be matched wherever its margin exceeds what fp32 can
move a score by."""
import numpy as np
import pytest
import torch

import oracle
from helpers import ATOL, RTOL, SCORE_RTOL, assert_attention_close
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _prompts(lens, Hkv, d, seed, outliers=True):
    """Concatenated bf16 prompt rows [T, Hkv, d] drawn N(0, 1), with a few
    (head, channel) pairs scaled x8 like the decode workloads' outliers."""
    g = torch.Generator().manual_seed(seed)
    T = int(sum(lens))
    k = torch.randn(T, Hkv, d, generator=g)
    v = torch.randn(T, Hkv, d, generator=g)
    if outliers:
        for _ in range(max(1, Hkv * d // 100)):
            h = int(torch.randint(Hkv, (1,), generator=g))
            c = int(torch.randint(d, (1,), generator=g))
            k[:, h, c] *= 8
            v[:, h, c] *= 8
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return k.to(torch.bfloat16), v.to(torch.bfloat16), cu


def _tables(kept, bs, seed, spare=3):
    """Block tables for the packed prompts (shuffled ids, -1 padding)."""
    rng = np.random.default_rng(seed)
    nb = [-(-int(n) // bs) for n in kept]
    MB = max(max(nb), 1)
    N = sum(nb) + spare
    perm = rng.permutation(N).astype(np.int32)
    bt = np.full((len(kept), MB), -1, np.int32)
    c = 0
    for b, n in enumerate(nb):
        bt[b, :n] = perm[c:c + n]
        c += n
    return bt, N


def _assert_rel(got, ref, tol, what):
    inf = np.isinf(ref)
    assert np.array_equal(np.isinf(got), inf), what
    g, r = got[~inf], ref[~inf]
    zero = r == 0
    assert (g[zero] == 0).all(), what
    rel = np.abs(g[~zero] - r[~zero]) / np.abs(r[~zero])
    assert rel.size == 0 or rel.max() <= tol, f"{what}: max rel err {rel.max():.3g}"


@pytest.mark.parametrize("Hkv,d", [(8, 128), (2, 64), (4, 256), (1, 64)])
def test_prefill_scores_match_oracle(Hkv, d):
    lens = [300, 1, 0, 1029, 77]
    k, v, cu = _prompts(lens, Hkv, d, seed=400 + d + Hkv)
    ref = oracle.prefill_scores(W.bits(k), W.bits(v))
    s = torch.full((k.shape[0],), float("nan"), device="cuda")
    pk.pe_prefill_scores(s, k.cuda(), v.cuda())
    torch.cuda.synchronize()
    _assert_rel(s.cpu().numpy().astype(np.float64), ref, SCORE_RTOL, f"Hkv={Hkv} d={d}")


def test_prefill_scores_zero_rules():
    """||K|| = 0 in every head: +inf when V is non-zero, 0 when V is zero too;
    one zero-K head among finite ones makes the head mean +inf."""
    Hkv, d = 4, 128
    k = torch.randn(3, Hkv, d).to(torch.bfloat16)
    v = torch.randn(3, Hkv, d).to(torch.bfloat16)
    k[0] = 0
    k[1] = 0
    v[1] = 0
    k[2, 2] = 0
    s = torch.empty(3, device="cuda")
    pk.pe_prefill_scores(s, k.cuda(), v.cuda())
    got = s.cpu().numpy()
    assert got[0] == np.inf and got[1] == 0.0 and got[2] == np.inf
    assert np.array_equal(got.astype(np.float64), oracle.prefill_scores(W.bits(k), W.bits(v)))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_prefill_select_bit_exact_with_ties(seed):
    """Seeded scores with many ties, infinities, NaN and signed zeros; prompt
    lengths below, at and above the budget, empty, and long (several passes of
    the 1024-thread compaction)."""
    rng = np.random.default_rng(900 + seed)
    budget = 700
    lens = [0, 5, 700, 701, 5000, 1, 40000, 1024, 2049]
    T = sum(lens)
    pool = np.array([0.0, -0.0, 1.0, 2.0, 0.5, np.inf, -np.inf, np.nan, -3.0, 1e-30, 7.25],
                    np.float32)
    scores = np.where(rng.random(T) < 0.5, rng.choice(pool, T),
                      rng.random(T).astype(np.float32) * 4).astype(np.float32)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    keep_ref, kept_ref = oracle.prefill_select(scores, cu, budget)
    B = len(lens)
    keep = torch.full((B, budget), -7, dtype=torch.int32, device="cuda")
    kept = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.pe_prefill_select(keep, kept, torch.as_tensor(scores).cuda(), torch.as_tensor(cu).cuda(),
                         err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert np.array_equal(kept.cpu().numpy(), kept_ref)
    assert np.array_equal(keep.cpu().numpy(), keep_ref)


def test_prefill_select_all_equal_and_monotone():
    budget = 100
    lens = [3000, 3000, 3000]
    s = np.concatenate([np.ones(3000), np.arange(3000), np.arange(3000)[::-1]]).astype(np.float32)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    keep = torch.empty(3, budget, dtype=torch.int32, device="cuda")
    kept = torch.empty(3, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.pe_prefill_select(keep, kept, torch.as_tensor(s).cuda(), torch.as_tensor(cu).cuda(), err)
    got = keep.cpu().numpy()
    last = np.arange(2900, 3000)
    assert np.array_equal(got[0], last) and np.array_equal(got[1], last)
    assert np.array_equal(got[2], np.arange(100))


@pytest.mark.parametrize("bs", [16, 256, 12, 1, 3, 8])
def test_prefill_pack_bit_exact(bs):
    """Keep sets from the oracle's select; packed pools compared byte for byte."""
    Hkv, d, budget = 8, 128, 300
    lens = [1000, 0, 299, 300, 301, 17]
    k, v, cu = _prompts(lens, Hkv, d, seed=31 + bs)
    kb, vb = W.bits(k), W.bits(v)
    keep_ref, kept_ref = oracle.prefill_select(oracle.prefill_scores(kb, vb), cu, budget)
    bt, N = _tables(kept_ref, bs, seed=bs)
    stride = bs * Hkv * d
    kc_ref = np.zeros(N * stride, np.uint16)
    vc_ref = np.zeros_like(kc_ref)
    oracle.prefill_pack(kb, vb, cu, keep_ref, kept_ref, kc_ref, vc_ref, stride, bt, bs)
    kc = torch.zeros(N, bs, Hkv, d, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.pe_prefill_pack(kc, vc, torch.as_tensor(bt).cuda(), k.cuda(), v.cuda(),
                       torch.as_tensor(cu).cuda(), torch.as_tensor(keep_ref).cuda(),
                       torch.as_tensor(kept_ref).cuda(), err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert np.array_equal(W.bits(kc).ravel(), kc_ref)
    assert np.array_equal(W.bits(vc).ravel(), vc_ref)


def _keep_consistent(keep_gpu, kept_gpu, scores_ref, cu, budget):
    """The GPU's keep set (decided on fp32 scores) against the oracle's fp64
    scores: same count; a token outranked by more than the fp32 margin at the
    threshold is evicted, one above it is kept.  Returns the number of prompts
    whose sets match the oracle's exactly."""
    keep_ref, kept_ref = oracle.prefill_select(scores_ref, cu, budget)
    assert np.array_equal(kept_gpu, kept_ref)
    exact = 0
    for b in range(len(cu) - 1):
        n = int(cu[b + 1] - cu[b])
        got = keep_gpu[b, :kept_gpu[b]]
        assert (np.diff(got) > 0).all() and (got >= 0).all() and (got < max(n, 1)).all()
        assert (keep_gpu[b, kept_gpu[b]:] == -1).all()
        ref = keep_ref[b, :kept_ref[b]]
        if np.array_equal(got, ref):
            exact += 1
            continue
        s = scores_ref[cu[b]:cu[b + 1]]
        tau = np.sort(s)[::-1][budget - 1]          # the oracle's threshold value
        margin = 4 * SCORE_RTOL * abs(tau)
        kept_mask = np.zeros(n, bool)
        kept_mask[got] = True
        assert kept_mask[s > tau + margin].all(), b
        assert not kept_mask[s < tau - margin].any(), b
    return exact


@pytest.mark.parametrize("bs", [16, 256, 5])
def test_prefill_compress_then_decode(bs):
    """One call scores, selects and packs; then a decode step over the
    compressed cache matches the oracle's decode over the oracle's packed pool."""
    Hkv, d, Hq, budget = 8, 128, 32, 512
    lens = [2000, 513, 512, 100, 0, 4100]
    k, v, cu = _prompts(lens, Hkv, d, seed=77 + bs)
    kb, vb = W.bits(k), W.bits(v)
    s_ref = oracle.prefill_scores(kb, vb)
    keep_ref, kept_ref = oracle.prefill_select(s_ref, cu, budget)
    bt, N = _tables(np.maximum(kept_ref, 1), bs, seed=5)
    B, T = len(lens), int(cu[-1])
    kc = torch.zeros(N, bs, Hkv, d, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    scores = torch.empty(T, device="cuda")
    keep = torch.empty(B, budget, dtype=torch.int32, device="cuda")
    kept = torch.empty(B, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt_d = torch.as_tensor(bt).cuda()
    pk.pe_prefill_compress(kc, vc, bt_d, k.cuda(), v.cuda(), torch.as_tensor(cu).cuda(), scores,
                           keep, kept, err)
    torch.cuda.synchronize()
    assert err.item() == 0
    _assert_rel(scores.cpu().numpy().astype(np.float64), s_ref, SCORE_RTOL, "compress scores")
    exact = _keep_consistent(keep.cpu().numpy(), kept.cpu().numpy(), s_ref, cu, budget)
    assert exact == B   # continuous N(0, 1) data at these sizes has no near-ties
    stride = bs * Hkv * d
    kc_ref = np.zeros(N * stride, np.uint16)
    vc_ref = np.zeros_like(kc_ref)
    oracle.prefill_pack(kb, vb, cu, keep_ref, kept_ref, kc_ref, vc_ref, stride, bt, bs)
    assert np.array_equal(W.bits(kc).ravel(), kc_ref)
    assert np.array_equal(W.bits(vc).ravel(), vc_ref)
    # decode over the compressed cache (sequences with at least one kept token)
    live = [b for b in range(B) if kept_ref[b] > 0]
    g = torch.Generator().manual_seed(3)
    q = torch.randn(len(live), Hq, d, generator=g).to(torch.bfloat16)
    ctx = torch.as_tensor(kept_ref[live]).cuda()
    btl = bt_d[live].contiguous()
    out = torch.empty(len(live), Hq, d, dtype=torch.bfloat16, device="cuda")
    ws = pk.alloc_workspace(len(live), Hq, Hkv, d, bs, bt.shape[1], 0, "cuda")
    pk.pa_decode(out, q.cuda(), kc, vc, btl, ctx, d ** -0.5, err, ws)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oracle.paged_decode(W.bits(q), kc_ref, vc_ref, stride, bt[live], kept_ref[live], Hkv,
                              bs, d ** -0.5)
    assert_attention_close(out, ref, "decode after prefill compression")


def test_prefill_compress_full_size_budget_1024():
    """The pages' 1024-token budget on 32 prompts of 8192 tokens in the
    Llama-3-8B KV shape (Hkv = 8, d = 128; 1 GiB of prompt rows): every score
    and every keep decision checked against the oracle."""
    Hkv, d, bs, budget = 8, 128, 16, 1024
    lens = [8192] * 32
    k, v, cu = _prompts(lens, Hkv, d, seed=1024)
    kb, vb = W.bits(k), W.bits(v)
    s_ref = oracle.prefill_scores(kb, vb)
    B, T = len(lens), int(cu[-1])
    bt, N = _tables([budget] * B, bs, seed=6)
    kc = torch.zeros(N, bs, Hkv, d, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    scores = torch.empty(T, device="cuda")
    keep = torch.empty(B, budget, dtype=torch.int32, device="cuda")
    kept = torch.empty(B, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kd, vd = k.cuda(), v.cuda()
    pk.pe_prefill_compress(kc, vc, torch.as_tensor(bt).cuda(), kd, vd, torch.as_tensor(cu).cuda(),
                           scores, keep, kept, err)
    torch.cuda.synchronize()
    assert err.item() == 0
    _assert_rel(scores.cpu().numpy().astype(np.float64), s_ref, SCORE_RTOL, "full-size scores")
    keep_h = keep.cpu().numpy()
    _keep_consistent(keep_h, kept.cpu().numpy(), s_ref, cu, budget)
    # data movement: sampled positions hold exactly the source rows the GPU kept
    rng = np.random.default_rng(8)
    for b, p in zip(rng.integers(0, B, 64), rng.integers(0, budget, 64)):
        blk = bt[b, p // bs]
        src = int(cu[b]) + int(keep_h[b, p])
        assert torch.equal(kc[blk, p % bs].cpu(), k[src])
        assert torch.equal(vc[blk, p % bs].cpu(), v[src])


def _random_tables(lens, bs, MB, N, seed):
    rng = np.random.default_rng(seed)
    perm = rng.permutation(N).astype(np.int32)
    bt = np.full((len(lens), MB), -1, np.int32)
    c = 0
    for b, n in enumerate(lens):
        m = -(-int(n) // bs)
        bt[b, :m] = perm[c:c + m]
        c += m
    return bt


@pytest.mark.parametrize("bs", [16, 256, 1, 5])
def test_evict_compact_bit_exact(bs):
    rng = np.random.default_rng(50 + bs)
    B, MB = 64, 80
    lens = rng.integers(0, MB * bs + 1, B).astype(np.int32)
    lens[:4] = [0, bs - 1, bs, MB * bs]
    nfull = lens // bs
    evict = np.where(nfull > 0, rng.integers(0, np.maximum(nfull, 1)), -1).astype(np.int32)
    evict[5] = -1
    evict[3] = nfull[3] - 1                        # the newest (last) block of a full table
    evict[6] = 0 if nfull[6] > 0 else -1
    N = int(sum(-(-int(n) // bs) for n in lens)) + 10
    bt = _random_tables(lens, bs, MB, N, seed=bs)
    bt_ref, len_ref, freed_ref = oracle.evict_compact(bt, lens, evict, bs)
    bt_d = torch.as_tensor(bt).cuda()
    len_d = torch.as_tensor(lens).cuda()
    freed = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.pe_evict_compact(bt_d, len_d, torch.as_tensor(evict).cuda(), bs, err, freed)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert np.array_equal(bt_d.cpu().numpy(), bt_ref)
    assert np.array_equal(len_d.cpu().numpy(), len_ref)
    assert np.array_equal(freed.cpu().numpy(), freed_ref)


def test_evict_compact_flags_non_full_block_and_leaves_it():
    bs = 16
    lens = np.array([40, 40, 16], np.int32)        # full blocks: 2, 2, 1
    evict = np.array([2, 1, 1], np.int32)          # 2 is the partial block; 1 valid; 1 invalid
    bt = np.array([[4, 1, 7], [0, 2, 3], [5, -1, -1]], np.int32)
    bt_ref, len_ref, freed_ref = oracle.evict_compact(bt, lens, evict, bs)
    bt_d = torch.as_tensor(bt).cuda()
    len_d = torch.as_tensor(lens).cuda()
    freed = torch.full((3,), -9, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.pe_evict_compact(bt_d, len_d, torch.as_tensor(evict).cuda(), bs, err, freed)
    torch.cuda.synchronize()
    assert err.item() == pk.PA_DEV_BAD_EVICT
    assert np.array_equal(bt_d.cpu().numpy(), bt_ref)
    assert np.array_equal(len_d.cpu().numpy(), len_ref)
    assert np.array_equal(freed.cpu().numpy(), freed_ref)
    assert freed_ref.tolist() == [-1, 2, -1]


def test_decode_eviction_round_trip_on_device():
    """Score, select and compact on the device, then decode: equal to the
    oracle decoding the oracle-compacted table over the unchanged pool."""
    cfg = W.scaled(W.CONFIGS["c2"], key="evict-rt", layers=1, batch=6,
                   old_lens=(1024, 300, 47, 16, 15, 513))
    wl = W.generate(cfg, "cpu")
    dev_bt = torch.as_tensor(wl.block_tables).cuda()
    ctx = torch.as_tensor(wl.old_lens).cuda()      # no append: score the cached tokens
    kp, vp = wl.k_pool[0].cuda(), wl.v_pool[0].cuda()
    B, MB, bs, Hkv, d = cfg.batch, wl.max_blocks, cfg.block_size, cfg.hkv, cfg.head_dim
    scores = torch.empty(B, MB * bs, Hkv, device="cuda")
    evict = torch.empty(B, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.pe_score_tokens(scores, kp, vp, dev_bt, ctx, err)
    pk.pe_select_evict_block(evict, scores, ctx, bs)
    freed = torch.empty(B, dtype=torch.int32, device="cuda")
    pk.pe_evict_compact(dev_bt, ctx, evict, bs, err, freed)
    q = wl.q[0].cuda()
    out = torch.empty(B, cfg.hq, d, dtype=torch.bfloat16, device="cuda")
    ws = pk.alloc_workspace(B, cfg.hq, Hkv, d, bs, MB, 0, "cuda")
    pk.pa_decode(out, q, kp, vp, dev_bt, ctx, wl.scale, err, ws)
    torch.cuda.synchronize()
    assert err.item() == 0
    # oracle: the same decision from its own scores (the gap guards near-ties)
    s = W.compact(wl, 0, range(B))
    stride = bs * Hkv * d
    kc, vc = s["k_pool"].ravel(), s["v_pool"].ravel()
    sc = oracle.score_tokens(kc, vc, stride, s["block_tables"], s["old_lens"], Hkv, d, bs)
    ev, means, gap = oracle.select_evict_block(sc, s["old_lens"], bs)
    assert np.array_equal(evict.cpu().numpy(), ev)
    bt_c, len_c, _ = oracle.evict_compact(s["block_tables"], s["old_lens"], ev, bs)
    assert np.array_equal(ctx.cpu().numpy(), len_c)
    ref = oracle.paged_decode(s["q"], kc, vc, stride, bt_c, len_c, Hkv, bs, wl.scale)
    assert_attention_close(out, ref, "decode after eviction")
