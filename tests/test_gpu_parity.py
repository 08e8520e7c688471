"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small and medium cases run the oracle on every output; they span several
16-token tiles, several partitions and ragged last blocks.  Append slots and
pool contents, INT8 codes and scales, and the evicted block are compared
exactly; attention within |err| <= 2e-3 + 1e-2 |ref|; scores within 1e-5
relative."""
import numpy as np
import pytest
import torch

import oracle

from helpers import (Device, assert_attention_close, assert_evict_consistent,
                     assert_scores_close, oracle_step)
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu

C = W.CONFIGS
MEDIUM = {
    # Llama-3.2-1B shape, 2 layers, 6 sequences around 1K tokens (ragged tails)
    "c2m": W.scaled(C["c2"], key="c2m", layers=2, batch=6, old_lens=(1024, 1000, 17, 300, 1,
                                                                      1039)),
    # Llama-3-8B shape with outlier channels, 7 sequences
    "c3m": W.scaled(C["c3"], key="c3m", layers=1, batch=7, old_len_range=(1, 900)),
    # nano-vLLM layout, block 256, no append
    "c4m": W.scaled(C["c4"], key="c4m", batch=3, old_lens=(4096, 3000, 257)),
    # INT8, G = 8
    "c5m": W.scaled(C["c5"], key="c5m", batch=5, old_lens=(300, 1, 16, 255, 512)),
    # block size 12 (not a multiple of 16): the general-shape kernel, with G = 16
    "bs12": W.scaled(C["c3"], key="bs12", layers=1, batch=4, hq=64, hkv=4, block_size=12,
                     old_len_range=(1, 700), outlier_frac=0.0),
    # G = 16 on the staged kernel, d = 64
    "g16": W.scaled(C["c2"], key="g16", layers=1, batch=3, hq=64, hkv=4, old_lens=(500, 33, 64)),
    # INT8 on the staged kernel with G = 16 and two 16-token sub-tiles per stage (Hkv = 4)
    "i8g16": W.scaled(C["c5"], key="i8g16", batch=3, hq=64, hkv=4, old_lens=(100, 37, 300)),
    # INT8 with d = 64: the general-shape kernel
    "i8d64": W.scaled(C["c5"], key="i8d64", batch=3, head_dim=64, old_lens=(70, 5, 200)),
    # FP8 (e4m3) pools: staged kernel (d = 128), G = 16 with two sub-tiles per stage, and the
    # general kernel (d = 64)
    "f8": W.scaled(C["c5"], key="f8", int8=False, fp8=True, batch=5,
                   old_lens=(300, 1, 16, 255, 512)),
    "f8g16": W.scaled(C["c5"], key="f8g16", int8=False, fp8=True, batch=3, hq=64, hkv=4,
                      old_lens=(100, 37, 300)),
    "f8d64": W.scaled(C["c5"], key="f8d64", int8=False, fp8=True, batch=3, head_dim=64,
                      old_lens=(70, 5, 200)),
}


def _parity(wl, layers, num_splits=0, score=None, pad=0):
    cfg = wl.cfg
    score = cfg.score if score is None else score
    seqs = range(cfg.batch)
    refs = [oracle_step(wl, l, seqs, score=score) for l in layers]
    dev = Device(wl, num_splits, pad=pad)
    if cfg.int8 or cfg.fp8:
        for l in layers:
            dev.fill_int8_history(l)
    for l, ref in zip(layers, refs):
        res = dev.step(l, score=score)
        torch.cuda.synchronize()
        assert dev.err.item() == 0, f"device error flag {dev.err.item()}"
        assert_attention_close(dev.out[l], ref["out"], f"{cfg.key} layer {l}")
        if "slots" in ref:
            # slots are global ids in the full pool; map the oracle's compact ids back
            s = ref["compact"]
            bt_full, bt_c = wl.block_tables, s["block_tables"]
            bs = cfg.block_size
            expect = np.empty_like(ref["slots"])
            for b in range(cfg.batch):
                blk, off = divmod(int(ref["slots"][b, 0]), bs)
                j = int(np.nonzero(bt_c[b] == blk)[0][0])
                expect[b, 0] = int(bt_full[b, j]) * bs + off
            assert np.array_equal(dev.slots.cpu().numpy(), expect)
        if score:
            lens = ref["ctx_lens"]
            got = res["scores"].cpu().numpy()
            for b in range(cfg.batch):
                assert_scores_close(got[b, :lens[b]], ref["scores"][b, :lens[b]], f"seq {b}")
            assert_evict_consistent(res["evict"].cpu().numpy(), ref["evict"], ref["means"],
                                    ref["gap"], cfg.key)
    return dev, refs


def test_tiny_workload_full_step():
    """[VKV] §2.1 append_slot and [KVL] "PagedEviction 块级驱逐机制" on the tiny workload:
    both pools after the append equal the oracle's bit for bit, and each sequence
    evicts exactly the oracle's block (its decision margins are large)."""
    wl = W.generate(C["c1"], "cpu")
    dev, refs = _parity(wl, [0], score=True)
    # pools after the append equal the oracle's, bit for bit (tiny pool: compare all of it)
    ref = refs[0]
    ids = torch.as_tensor(wl.block_tables[wl.block_tables >= 0], device="cuda")
    for pool, key in ((dev.k_pool, "kc"), (dev.v_pool, "vc")):
        got = pool[0][ids].view(torch.int16).cpu().numpy()
        assert np.array_equal(got.view(np.uint16).ravel(), ref[key]), key
    # 38 -> 2 full blocks, 101 -> 6 full blocks; the rest are not candidates
    assert (ref["means"][0, 2:] != ref["means"][0, 2:]).all()
    assert (ref["means"][1, 6:] != ref["means"][1, 6:]).all()
    assert ((ref["evict"] >= 0) & (ref["evict"] < [2, 6])).all()
    # the choice is unconditional here: the gap to the runner-up is far above what
    # 1e-5-relative scores can move a block mean by
    assert (ref["gap"] > 1e-3).all()
    got_evict = torch.full((2,), -9, dtype=torch.int32, device="cuda")
    scores = torch.empty(2, wl.max_blocks * 16, C["c1"].hkv, dtype=torch.float32, device="cuda")
    pk.pe_score_tokens(scores, dev.k_pool[0], dev.v_pool[0], dev.bt, dev.ctx, dev.err)
    pk.pe_select_evict_block(got_evict, scores, dev.ctx, 16)
    torch.cuda.synchronize()
    assert dev.err.item() == 0
    assert got_evict.cpu().numpy().tolist() == ref["evict"].tolist()


@pytest.mark.parametrize("key", list(MEDIUM))
def test_medium_workloads(key):
    wl = W.generate(MEDIUM[key], "cpu")
    _parity(wl, list(range(wl.q.shape[0])), score=(key == "c2m"))


@pytest.mark.parametrize("num_splits", [1, 2, 3, 8, 0, 96])
@pytest.mark.parametrize("kv", ["bf16", "bf16-d64", "bf16-g16", "int8", "fp8"])
def test_split_count_invariance(num_splits, kv):
    """num_splits = 96 cuts the 2000-token sequence into more than 32 partitions, the
    range where the merge splits the partials across the CTA's warps; with Hkv = 4
    (bf16-g16) each partition also leaves two partials per kv head."""
    base = {"bf16": C["c3"], "bf16-d64": C["c2"], "bf16-g16": C["c3"]}.get(kv, C["c5"])
    cfg = W.scaled(base, key="split", layers=1, batch=3, old_lens=(2000, 700, 45), score=False)
    if kv == "bf16-g16":
        cfg = W.scaled(cfg, hq=64, hkv=4)
    if kv == "fp8":
        cfg = W.scaled(cfg, int8=False, fp8=True)
    wl = W.generate(cfg, "cpu")
    _parity(wl, [0], num_splits=num_splits)


@pytest.mark.parametrize("kv", ["bf16", "int8", "fp8"])
def test_padded_block_stride(kv):
    """Pools whose blocks sit (bs + 3)·Hkv·d elements apart (views of a larger buffer
    whose gaps hold NaN, code 127 or the e4m3 NaN code): the history and new-token
    appends, the decode and the score match the oracle on dense pools, and no gap
    element is read or written."""
    base = C["c3"] if kv == "bf16" else C["c5"]
    cfg = W.scaled(base, key="pad", layers=1, batch=4, old_lens=(700, 45, 16, 1),
                   score=(kv == "bf16"))
    if kv == "fp8":
        cfg = W.scaled(cfg, int8=False, fp8=True)
    wl = W.generate(cfg, "cpu")
    dev, refs = _parity(wl, [0], pad=3)
    assert dev.pads_untouched()
    pool = {"bf16": "k_pool", "int8": "kq", "fp8": "k8"}[kv]
    N, bs, Hkv, d = getattr(dev, pool)[0].shape
    assert getattr(dev, pool)[0].stride(0) == (bs + 3) * Hkv * d


def test_physical_block_permutation_gives_identical_output():
    cfg = W.scaled(C["c2"], key="perm", layers=1, batch=4, old_lens=(100, 77, 300, 5))
    wl = W.generate(cfg, "cpu")
    dev = Device(wl)
    dev.step(0)
    base = dev.out[0].clone()
    N = wl.num_blocks
    perm = torch.randperm(N, generator=torch.Generator().manual_seed(1))
    inv = torch.argsort(perm)
    bt = torch.as_tensor(wl.block_tables)
    dev.bt = torch.where(bt >= 0, perm[bt.clamp(min=0)], bt).to(torch.int32).cuda()
    dev.k_pool[0] = dev.k_pool[0][inv.cuda()]
    dev.v_pool[0] = dev.v_pool[0][inv.cuda()]
    # the append already ran: decode only
    pk.pa_decode(dev.out[0], dev.q[0], dev.k_pool[0], dev.v_pool[0], dev.bt, dev.ctx, wl.scale,
                 dev.err, dev.ws)
    torch.cuda.synchronize()
    assert dev.err.item() == 0
    assert torch.equal(dev.out[0], base)


def test_unused_blocks_and_slots_are_never_read():
    cfg = W.scaled(C["c3"], key="nan", layers=1, batch=3, old_lens=(33, 1, 500), spare=0.5)
    wl = W.generate(cfg, "cpu")
    ref = oracle_step(wl, 0, range(3))
    used = set(wl.block_tables[wl.block_tables >= 0].tolist())
    unused = [p for p in range(wl.num_blocks) if p not in used]
    wl.k_pool[0, unused] = float("nan")
    wl.v_pool[0, unused] = float("nan")
    for b in range(3):   # slots past the new token in each last block
        n = int(wl.ctx_lens[b])
        last = wl.block_tables[b, (n - 1) // 16]
        if n % 16:
            wl.k_pool[0, last, n % 16:] = float("nan")
            wl.v_pool[0, last, n % 16:] = float("nan")
    dev = Device(wl)
    dev.step(0)
    torch.cuda.synchronize()
    assert dev.err.item() == 0
    assert_attention_close(dev.out[0], ref["out"], "nan-poisoned unused memory")


def test_deterministic_bitwise():
    cfg = W.scaled(C["c3"], key="det", layers=1, batch=5, old_len_range=(100, 3000))
    wl = W.generate(cfg, "cpu")
    dev = Device(wl)
    dev.step(0)
    a = dev.out[0].clone()
    pk.pa_decode(dev.out[0], dev.q[0], dev.k_pool[0], dev.v_pool[0], dev.bt, dev.ctx, wl.scale,
                 dev.err, dev.ws)
    torch.cuda.synchronize()
    assert torch.equal(a, dev.out[0])


@pytest.mark.parametrize("kv", ["bf16", "int8"])
def test_workspace_reuse_across_calls_with_other_partitions(kv):
    """The staged kernel's plan, unit list and partials live in the caller's workspace
    and are rewritten every call.  One workspace (filled with 0xff first) serves calls
    whose lengths give different partition counts; every call matches the oracle."""
    base = C["c3"] if kv == "bf16" else C["c5"]
    c1 = W.scaled(base, key="reuse1", layers=1, batch=4, old_lens=(2500, 40, 900, 1))
    c2 = W.scaled(base, key="reuse2", layers=1, batch=4, old_lens=(7, 2500, 64, 1300))
    w1, w2 = W.generate(c1, "cpu"), W.generate(c2, "cpu")
    r1, r2 = oracle_step(w1, 0, range(4)), oracle_step(w2, 0, range(4))
    d1, d2 = Device(w1), Device(w2)
    n = max(d1.ws.numel(), d2.ws.numel())
    ws = torch.full((n,), 0xFF, dtype=torch.uint8, device="cuda")
    d1.ws = d2.ws = ws
    if kv == "int8":
        d1.fill_int8_history(0)
        d2.fill_int8_history(0)
    for dev, ref, tag in ((d1, r1, "first"), (d2, r2, "second"), (d1, r1, "third")):
        dev.step(0)
        torch.cuda.synchronize()
        assert dev.err.item() == 0
        assert_attention_close(dev.out[0], ref["out"], f"{kv} {tag} call")


def test_int8_codes_and_scales_bit_exact():
    wl = W.generate(MEDIUM["c5m"], "cpu")
    ref = oracle_step(wl, 0, range(wl.cfg.batch))
    dev = Device(wl)
    dev.fill_int8_history(0)
    dev.step(0)
    torch.cuda.synchronize()
    ids = torch.as_tensor(wl.block_tables[wl.block_tables >= 0], device="cuda")
    assert np.array_equal(dev.kq[0][ids].cpu().numpy().ravel(), ref["kq"])
    assert np.array_equal(dev.vq[0][ids].cpu().numpy().ravel(), ref["vq"])
    assert np.array_equal(dev.ks[0][ids].cpu().numpy().ravel(), ref["ks"])
    assert np.array_equal(dev.vs[0][ids].cpu().numpy().ravel(), ref["vs"])


def test_empty_batch_and_zero_length_context():
    cfg = W.scaled(C["c2"], key="zero", layers=1, batch=3, old_lens=(40, 0, 16))
    wl = W.generate(cfg, "cpu")
    dev = Device(wl)
    # sequence 1 attends to nothing: give it length 0 explicitly (no append for it)
    dev.ctx[1] = 0
    pk.pa_decode(dev.out[0], dev.q[0], dev.k_pool[0], dev.v_pool[0], dev.bt, dev.ctx, wl.scale,
                 dev.err, dev.ws)
    torch.cuda.synchronize()
    assert dev.err.item() == 0
    assert (dev.out[0, 1] == 0).all()
    # B = 0 is a no-op that succeeds
    pk.pa_decode(dev.out[0, :0], dev.q[0, :0], dev.k_pool[0], dev.v_pool[0], dev.bt[:0],
                 dev.ctx[:0], wl.scale, dev.err, dev.ws)


def test_device_flags_on_bad_table_and_length():
    cfg = W.scaled(C["c2"], key="bad", layers=1, batch=2, old_lens=(100, 50))
    wl = W.generate(cfg, "cpu")
    dev = Device(wl)
    bt = dev.bt.clone()
    bt[0, 2] = wl.num_blocks + 5        # a needed entry out of range
    pk.pa_decode(dev.out[0], dev.q[0], dev.k_pool[0], dev.v_pool[0], bt, dev.ctx, wl.scale,
                 dev.err, dev.ws)
    torch.cuda.synchronize()
    assert dev.err.item() & pk.PA_DEV_BAD_BLOCK
    dev.err.zero_()
    ctx = dev.ctx.clone()
    ctx[1] = wl.max_blocks * 16 + 1     # longer than the table can hold
    pk.pa_decode(dev.out[0], dev.q[0], dev.k_pool[0], dev.v_pool[0], dev.bt, ctx, wl.scale,
                 dev.err, dev.ws)
    torch.cuda.synchronize()
    assert dev.err.item() & pk.PA_DEV_BAD_LEN
    assert (dev.out[0, 1] == 0).all()
    dev.err.zero_()
    pos = dev.pos.clone()
    pos[0] = wl.max_blocks * 16         # append position past the table
    pk.pa_append_kv(dev.k_new[0], dev.v_new[0], dev.k_pool[0], dev.v_pool[0], dev.bt, pos,
                    dev.err, slot_out=dev.slots)
    torch.cuda.synchronize()
    assert dev.err.item() & pk.PA_DEV_BAD_LEN
    assert dev.slots[0, 0].item() == -1


def test_select_evict_bit_exact_on_given_scores():
    """a5 alone: on the same fp32 scores both sides take the decision in fp64, so
    the means (rounded to fp32) and the chosen block agree exactly."""
    rng = np.random.default_rng(5)
    B, MB, bs, Hkv = 9, 33, 16, 8
    scores = rng.uniform(0.5, 2.0, (B, MB * bs, Hkv)).astype(np.float32)
    lens = np.array([0, 15, 16, 17, 100, 528, 500, 333, 48], np.int32)
    scores[4, 32:48] = 0.4   # planted low block 2 of sequence 4
    scores[8, :] = 1.25      # all equal: lowest index
    ev, means, gap = __import__("oracle").select_evict_block(scores, lens, bs)
    evict = torch.empty(B, dtype=torch.int32, device="cuda")
    gm = torch.empty(B, MB, dtype=torch.float32, device="cuda")
    pk.pe_select_evict_block(evict, torch.as_tensor(scores).cuda(), torch.as_tensor(lens).cuda(),
                             bs, gm)
    torch.cuda.synchronize()
    assert evict.cpu().numpy().tolist() == ev.tolist()
    assert ev[4] == 2 and ev[8] == 0 and ev[0] == -1 and ev[1] == -1
    gmn = gm.cpu().numpy()
    assert np.array_equal(np.isnan(gmn), np.isnan(means))
    ok = ~np.isnan(means)
    assert np.array_equal(gmn[ok], means[ok].astype(np.float32))


def test_fp8_codes_bit_exact():
    wl = W.generate(MEDIUM["f8"], "cpu")
    ref = oracle_step(wl, 0, range(wl.cfg.batch))
    dev = Device(wl)
    dev.fill_int8_history(0)
    dev.step(0)
    torch.cuda.synchronize()
    ids = torch.as_tensor(wl.block_tables[wl.block_tables >= 0], device="cuda")
    assert np.array_equal(dev.k8[0][ids].cpu().numpy().ravel(), ref["k8"])
    assert np.array_equal(dev.v8[0][ids].cpu().numpy().ravel(), ref["v8"])


def test_fp8_append_special_values_bit_exact():
    """Saturation beyond 448 (and of infinities), NaN, signed zero, subnormal
    steps and ties to even on both sides of the subnormal/normal boundary."""
    Hkv, d, bs, N = 2, 128, 16, 4
    special = [0.0, -0.0, 448.0, -448.0, 449.0, 464.0, 480.0, 1e4, -1e4, float("inf"),
               float("-inf"), float("nan"), 2.0 ** -9, 3 * 2.0 ** -10, 2.0 ** -10,
               5 * 2.0 ** -10, 2.0 ** -6, 15 * 2.0 ** -10, 17 * 2.0 ** -10, 1.0625, 1.1875,
               -1.0625, 240.0, 248.0, 232.0, 0.001, -0.0029296875]
    g = torch.Generator().manual_seed(17)
    k = torch.randn(1, 3, Hkv, d, generator=g) * 40
    flat = k.view(-1)
    flat[:len(special)] = torch.tensor(special)
    neg = [-x for x in special if x == x]   # NaN once only: its sign is not a defined result
    flat[-len(neg):] = torch.tensor(neg)
    k = k.to(torch.bfloat16)
    v = (torch.randn(1, 3, Hkv, d, generator=g) * 0.01).to(torch.bfloat16)
    k8 = torch.zeros(N, bs, Hkv, d, dtype=torch.uint8, device="cuda")
    v8 = torch.zeros_like(k8)
    bt = torch.tensor([[2, 0]], dtype=torch.int32, device="cuda")
    pos = torch.tensor([14], dtype=torch.int32, device="cuda")   # rows 14, 15 of block 2, row 0 of block 0
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.pa_append_kv_fp8(k.cuda(), v.cuda(), k8, v8, bt, pos, err)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = torch.stack([k8[2, 14], k8[2, 15], k8[0, 0]]).cpu().numpy().ravel()
    expect = oracle.quantize_e4m3(W.bits(k)).ravel()
    assert np.array_equal(got, expect)
    gotv = torch.stack([v8[2, 14], v8[2, 15], v8[0, 0]]).cpu().numpy().ravel()
    assert np.array_equal(gotv, oracle.quantize_e4m3(W.bits(v)).ravel())
    # nothing else in the pools was touched
    assert int(k8.count_nonzero()) == int(np.count_nonzero(got))


def wide_range_queries(q: torch.Tensor, seed: int) -> torch.Tensor:
    """Query rows whose magnitudes span the bf16 range, one kind per query head
    (cycling): a row mixing 3e4, N(0,1) and 1e-4 elements; a row scaled by 1e5
    (every element beyond fp16's 65504 for most); per-element magnitudes 2^-20 ..
    2^12; N(0,1) rows scaled by 10, 30, 300 and 1e-30; one element of 7e4 among
    N(0,1).  The page's INT8 and FP8 caches quantise K and V only ([VKV] §6.1
    quantize_kv_cache); the query stays bf16, so every bf16 row is a valid input."""
    g = torch.Generator().manual_seed(seed)
    L, B, Hq, d = q.shape
    out = torch.randn(L, B, Hq, d, generator=g, dtype=torch.float64)
    for i in range(Hq):
        kind = i % 8
        r = out[:, :, i]
        if kind == 0:
            r[..., 0] = 3e4
            r[..., d // 3:] *= 1e-4
            perm = torch.randperm(d, generator=g)
            out[:, :, i] = r[..., perm]
        elif kind == 1:
            r *= 1e5
        elif kind == 2:
            e = torch.randint(-20, 13, r.shape, generator=g).double()
            r.copy_(torch.sign(r) * torch.pow(2.0, e) * (1 + torch.rand(r.shape, generator=g,
                                                                       dtype=torch.float64)))
        elif kind == 3:
            r *= 10
        elif kind == 4:
            r *= 30
        elif kind == 5:
            r *= 300
        elif kind == 6:
            r *= 1e-30
        else:
            r[..., 5] = -7e4
    return out.to(torch.bfloat16)


def _stored_kv(ref, cfg):
    """The K and V values the oracle attended, per compacted sequence: float64
    [len, Hkv, d] arrays gathered through the compacted block table."""
    s = ref["compact"]
    bs, Hkv, d = cfg.block_size, cfg.hkv, cfg.head_dim
    if cfg.fp8:
        dec = lambda c: torch.from_numpy(c).view(torch.float8_e4m3fn).double().numpy()
        k, v = dec(ref["k8"]), dec(ref["v8"])
    elif cfg.int8:
        k = ref["kq"].astype(np.float64) * np.repeat(ref["ks"].astype(np.float64), d)
        v = ref["vq"].astype(np.float64) * np.repeat(ref["vs"].astype(np.float64), d)
    else:
        tobf = lambda c: torch.from_numpy(c.view(np.int16)).view(torch.bfloat16).double().numpy()
        k, v = tobf(ref["kc"]), tobf(ref["vc"])
    k = k.reshape(-1, bs, Hkv, d)
    v = v.reshape(-1, bs, Hkv, d)
    out = []
    for b, n in enumerate(ref["ctx_lens"]):
        blocks = s["block_tables"][b, :(int(n) + bs - 1) // bs]
        out.append((k[blocks].reshape(-1, Hkv, d)[:n], v[blocks].reshape(-1, Hkv, d)[:n]))
    return out


def fp32_logit_slack(q, kv, G, scale):
    """Per (sequence, query head): the output error that the logits' fp32 resolution
    alone allows.  A logit of magnitude |s| is held to about 2^-24 |s|, and the
    tensor-core accumulation of a k-step aligns its products to the largest, so a
    row whose logits are huge (a query element of 7e4, or every element 1e5) carries
    a few ulps of that magnitude: Delta = 2^-22 max_t |scale s_t|.  Weights move by
    a factor within e^(+-Delta), so the output moves by at most 2 Delta max_t |v_t|.
    For N(0,1) rows this is below 1e-5; the fp64 oracle has no such limit."""
    B, Hq, d = q.shape
    slack = np.zeros((B, Hq, 1))
    for b in range(B):
        k, v = kv[b]
        if len(k) == 0:
            continue
        for i in range(Hq):
            s = k[:, i // G, :] @ q[b, i].astype(np.float64)
            slack[b, i, 0] = 2.0 * 2.0 ** -22 * np.abs(s * scale).max() * np.abs(v[:, i // G]).max()
    return slack


@pytest.mark.parametrize("key", ["c5m", "i8g16", "i8d64", "f8", "f8g16", "f8d64", "c3m", "c2m"])
def test_wide_range_queries(key):
    """INT8 (three-part int8 query on the staged kernel), FP8 (power-of-two prescaled fp16
    query), bf16 and the general kernels against the fp64 oracle on queries whose
    magnitudes span the bf16 range; no device flag is raised.  The tolerance adds, per
    row, what the logits' fp32 resolution allows (fp32_logit_slack; negligible except
    for rows whose logits run into the tens of thousands)."""
    cfg = W.scaled(MEDIUM[key], score=False)
    wl = W.generate(cfg, "cpu")
    wl.q.copy_(wide_range_queries(wl.q, 396 + len(key)))
    assert wl.q.float().abs().max() > 65504
    layers = list(range(wl.q.shape[0]))
    refs = [oracle_step(wl, l, range(cfg.batch)) for l in layers]
    dev = Device(wl)
    if cfg.int8 or cfg.fp8:
        for l in layers:
            dev.fill_int8_history(l)
    for l, ref in zip(layers, refs):
        dev.step(l)
        torch.cuda.synchronize()
        assert dev.err.item() == 0, f"device error flag {dev.err.item()}"
        got = dev.out[l].float().cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        q = wl.q[l].double().numpy()
        slack = fp32_logit_slack(q, _stored_kv(ref, cfg), cfg.hq // cfg.hkv, wl.scale)
        err = np.abs(got - ref["out"])
        bound = 2e-3 + 1e-2 * np.abs(ref["out"]) + slack
        bad = err > bound
        assert not bad.any(), (f"{key} layer {l}: {bad.sum()} outside; worst excess "
                               f"{(err - bound).max():.3g}; slack range {slack.min():.2g}.."
                               f"{slack.max():.2g}")
