"""Pools beyond 2^31 elements.

One layer's pool on a 180 GB device can hold tens of GB.  The sequences' blocks then
sit at physical ids whose element offsets pass 2^31, so every offset a kernel forms
from a block id (slot = block_table[pos / bs] * bs + pos % bs, [VKV] §2.1; the
gather of [KVP] "PagedAttention 的算子") must be 64-bit.  Each kernel that addresses a
pool runs here on such a pool, whose used blocks sit at ids from ceil(2^31 / block
elements) on and whose other blocks hold NaN (NaN scales, NaN e4m3 codes).  It also
runs on a small pool holding the same blocks at low ids.  A paged result depends
only on the block table's logical order, so the two must agree bit for bit.  The
decode outputs also match the fp64 oracle on the small pool."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_attention_close
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu

BS, HKV, HQ = 16, 8, 32
LENS = [37, 300, 1000]   # tokens cached per sequence before the appended one
STEP = 7                 # big-pool id = base + STEP * small id


def _tables(seed):
    """Shuffled block tables over a small pool, with room for one appended token."""
    rng = np.random.default_rng(seed)
    nb = [-(-(n + 1) // BS) for n in LENS]
    n_small = sum(nb) + 3
    perm = rng.permutation(n_small).astype(np.int32)
    bt = np.full((len(LENS), max(nb)), -1, np.int32)
    c = 0
    for b, m in enumerate(nb):
        bt[b, :m] = perm[c:c + m]
        c += m
    return bt, n_small


def _layout(block_elems, n_small):
    """First block id whose element offset reaches 2^31, and the big pool's size."""
    base = -(-(1 << 31) // block_elems)
    assert base * block_elems >= 1 << 31
    return base, base + STEP * n_small


def _place(small, n_big, base, fill):
    """A pool of n_big blocks, all `fill`, with small's blocks at base + STEP * id."""
    big = torch.full((n_big,) + tuple(small.shape[1:]), fill, dtype=small.dtype,
                     device=small.device)
    ids = torch.arange(small.shape[0], device=small.device) * STEP + base
    big[ids] = small
    return big, ids


def _same_bits(a, b, what):
    if a.dtype.is_floating_point:
        a = a.view(torch.int16 if a.element_size() == 2 else torch.int32)
        b = b.view(a.dtype)
    assert torch.equal(a, b), what


def _common(seed, d, dev="cuda"):
    g = torch.Generator().manual_seed(seed)
    bt, n_small = _tables(seed)
    B = len(LENS)
    pos = torch.as_tensor(LENS, dtype=torch.int32, device=dev)
    x = dict(
        g=g, bt=bt, n_small=n_small, B=B, pos=pos, ctx=pos + 1,
        k_new=torch.randn(B, HKV, d, generator=g).to(torch.bfloat16).to(dev),
        v_new=torch.randn(B, HKV, d, generator=g).to(torch.bfloat16).to(dev),
        q=torch.randn(B, HQ, d, generator=g).to(torch.bfloat16).to(dev),
        scale=d ** -0.5)
    return x


@pytest.mark.parametrize("d", [64, 128])
def test_bf16_append_score_and_decode_beyond_2_31_elements(d):
    dev = "cuda"
    x = _common(900 + d, d)
    base, n_big = _layout(BS * HKV * d, x["n_small"])
    ks = torch.randn(x["n_small"], BS, HKV, d, generator=x["g"]).to(torch.bfloat16).to(dev)
    vs = torch.randn(x["n_small"], BS, HKV, d, generator=x["g"]).to(torch.bfloat16).to(dev)
    kb, ids = _place(ks, n_big, base, float("nan"))
    vb, _ = _place(vs, n_big, base, float("nan"))
    bt_s = torch.as_tensor(x["bt"], device=dev)
    bt_b = torch.as_tensor(np.where(x["bt"] >= 0, base + STEP * x["bt"], -1).astype(np.int32),
                           device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    B = x["B"]
    slot_s = torch.empty(B, 1, dtype=torch.int64, device=dev)
    slot_b = torch.empty_like(slot_s)
    pk.pa_append_kv(x["k_new"], x["v_new"], ks, vs, bt_s, x["pos"], err, slot_out=slot_s)
    pk.pa_append_kv(x["k_new"], x["v_new"], kb, vb, bt_b, x["pos"], err, slot_out=slot_b)
    torch.cuda.synchronize()
    assert err.item() == 0
    s = slot_s.cpu().numpy()
    assert np.array_equal(slot_b.cpu().numpy(), (base + STEP * (s // BS)) * BS + s % BS)
    _same_bits(kb[ids], ks, "K blocks after the append")
    _same_bits(vb[ids], vs, "V blocks after the append")

    # decode over the big pool: the same bits as over the small one, and the oracle
    MB = x["bt"].shape[1]
    outs = []
    for kc, vc, bt in ((ks, vs, bt_s), (kb, vb, bt_b)):
        out = torch.full_like(x["q"], float("nan"))
        ws = pk.alloc_workspace(B, HQ, HKV, d, BS, MB, 0, dev)
        pk.pa_decode(out, x["q"], kc, vc, bt, x["ctx"], x["scale"], err, ws)
        outs.append(out)
    torch.cuda.synchronize()
    assert err.item() == 0
    _same_bits(outs[1], outs[0], "decode output")
    ref = oracle.paged_decode(W.bits(x["q"]), W.bits(ks).ravel(), W.bits(vs).ravel(),
                              BS * HKV * d, x["bt"], x["ctx"].cpu().numpy(), HKV, BS,
                              x["scale"])
    assert_attention_close(outs[1], ref, f"decode over a pool past 2^31 elements, d {d}")

    # norm-ratio scores read through the same block ids
    scores = []
    for kc, vc, bt in ((ks, vs, bt_s), (kb, vb, bt_b)):
        sc = torch.zeros(B, MB * BS, HKV, dtype=torch.float32, device=dev)
        pk.pe_score_tokens(sc, kc, vc, bt, x["ctx"], err)
        scores.append(sc)
    torch.cuda.synchronize()
    assert err.item() == 0
    _same_bits(scores[1], scores[0], "token scores")


def test_int8_append_and_decode_beyond_2_31_elements():
    dev, d = "cuda", 128
    x = _common(1200, d)
    base, n_big = _layout(BS * HKV * d, x["n_small"])
    g = x["g"]
    shape = (x["n_small"], BS, HKV, d)
    kq = torch.randint(-127, 128, shape, generator=g, dtype=torch.int8).to(dev)
    vq = torch.randint(-127, 128, shape, generator=g, dtype=torch.int8).to(dev)
    ksc = (torch.rand(shape[:3], generator=g) * 0.02 + 0.001).to(dev)
    vsc = (torch.rand(shape[:3], generator=g) * 0.02 + 0.001).to(dev)
    kqb, ids = _place(kq, n_big, base, 0)
    vqb, _ = _place(vq, n_big, base, 0)
    kscb, _ = _place(ksc, n_big, base, float("nan"))
    vscb, _ = _place(vsc, n_big, base, float("nan"))
    bt_s = torch.as_tensor(x["bt"], device=dev)
    bt_b = torch.as_tensor(np.where(x["bt"] >= 0, base + STEP * x["bt"], -1).astype(np.int32),
                           device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pk.pa_append_kv_int8(x["k_new"], x["v_new"], kq, vq, ksc, vsc, bt_s, x["pos"], err)
    pk.pa_append_kv_int8(x["k_new"], x["v_new"], kqb, vqb, kscb, vscb, bt_b, x["pos"], err)
    torch.cuda.synchronize()
    assert err.item() == 0
    _same_bits(kqb[ids], kq, "K codes")
    _same_bits(vqb[ids], vq, "V codes")
    _same_bits(kscb[ids], ksc, "K scales")
    _same_bits(vscb[ids], vsc, "V scales")
    B, MB = x["B"], x["bt"].shape[1]
    outs = []
    for pools, bt in (((kq, vq, ksc, vsc), bt_s), ((kqb, vqb, kscb, vscb), bt_b)):
        out = torch.full_like(x["q"], float("nan"))
        ws = pk.alloc_workspace(B, HQ, HKV, d, BS, MB, 0, dev)
        pk.pa_decode_int8(out, x["q"], *pools, bt, x["ctx"], x["scale"], err, ws)
        outs.append(out)
    torch.cuda.synchronize()
    assert err.item() == 0
    _same_bits(outs[1], outs[0], "INT8 decode output")
    ref = oracle.paged_decode_int8(W.bits(x["q"]), kq.cpu().numpy().ravel(),
                                   vq.cpu().numpy().ravel(), ksc.cpu().numpy().ravel(),
                                   vsc.cpu().numpy().ravel(), BS * HKV * d, x["bt"],
                                   x["ctx"].cpu().numpy(), HKV, BS, x["scale"])
    assert_attention_close(outs[1], ref, "INT8 decode over a pool past 2^31 elements")


def test_fp8_append_and_decode_beyond_2_31_elements():
    dev, d = "cuda", 128
    x = _common(1300, d)
    base, n_big = _layout(BS * HKV * d, x["n_small"])
    shape = (x["n_small"], BS, HKV, d)
    # finite e4m3 codes only in the blocks in use (0x7f / 0xff are NaN)
    k8 = torch.randint(0, 0x7f, shape, generator=x["g"], dtype=torch.int64)
    v8 = torch.randint(0, 0x7f, shape, generator=x["g"], dtype=torch.int64)
    sign = torch.randint(0, 2, shape, generator=x["g"], dtype=torch.int64) * 0x80
    k8 = (k8 | sign).to(torch.uint8).to(dev)
    v8 = (v8 | sign.flip(0)).to(torch.uint8).to(dev)
    k8b, ids = _place(k8, n_big, base, 0x7f)
    v8b, _ = _place(v8, n_big, base, 0x7f)
    bt_s = torch.as_tensor(x["bt"], device=dev)
    bt_b = torch.as_tensor(np.where(x["bt"] >= 0, base + STEP * x["bt"], -1).astype(np.int32),
                           device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pk.pa_append_kv_fp8(x["k_new"], x["v_new"], k8, v8, bt_s, x["pos"], err)
    pk.pa_append_kv_fp8(x["k_new"], x["v_new"], k8b, v8b, bt_b, x["pos"], err)
    torch.cuda.synchronize()
    assert err.item() == 0
    _same_bits(k8b[ids], k8, "K codes")
    _same_bits(v8b[ids], v8, "V codes")
    B, MB = x["B"], x["bt"].shape[1]
    outs = []
    for kc, vc, bt in ((k8, v8, bt_s), (k8b, v8b, bt_b)):
        out = torch.full_like(x["q"], float("nan"))
        ws = pk.alloc_workspace(B, HQ, HKV, d, BS, MB, 0, dev)
        pk.pa_decode_fp8(out, x["q"], kc, vc, bt, x["ctx"], x["scale"], err, ws)
        outs.append(out)
    torch.cuda.synchronize()
    assert err.item() == 0
    _same_bits(outs[1], outs[0], "FP8 decode output")
    ref = oracle.paged_decode_fp8(W.bits(x["q"]), k8.cpu().numpy().ravel(),
                                  v8.cpu().numpy().ravel(), BS * HKV * d, x["bt"],
                                  x["ctx"].cpu().numpy(), HKV, BS, x["scale"])
    assert_attention_close(outs[1], ref, "FP8 decode over a pool past 2^31 elements")


@pytest.mark.parametrize("balanced", [False, True])
def test_chunked_prefill_attention_beyond_2_31_elements(balanced):
    """The tcgen05 multi-query kernel (d = 128) gathers its K/V tiles by TMA through
    the block table: the last 300 and 130 tokens of two sequences as query chunks."""
    dev, d = "cuda", 128
    x = _common(1400, d)
    base, n_big = _layout(BS * HKV * d, x["n_small"])
    g = x["g"]
    ks = torch.randn(x["n_small"], BS, HKV, d, generator=g).to(torch.bfloat16).to(dev)
    vs = torch.randn(x["n_small"], BS, HKV, d, generator=g).to(torch.bfloat16).to(dev)
    kb, _ = _place(ks, n_big, base, float("nan"))
    vb, _ = _place(vs, n_big, base, float("nan"))
    bt_s = torch.as_tensor(x["bt"], device=dev)
    bt_b = torch.as_tensor(np.where(x["bt"] >= 0, base + STEP * x["bt"], -1).astype(np.int32),
                           device=dev)
    lens = np.asarray(LENS, np.int32)
    qlens = [min(n, c) for n, c in zip(LENS, (37, 300, 130))]
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = torch.randn(int(cu[-1]), HQ, d, generator=g).to(torch.bfloat16).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    outs = []
    for kc, vc, bt in ((ks, vs, bt_s), (kb, vb, bt_b)):
        out = torch.full_like(q, float("nan"))
        ws = (pk.alloc_prefill_workspace(len(LENS), HQ, HKV, d, BS, max(qlens), dev)
              if balanced else None)
        pk.pa_prefill_attention(out, q, torch.as_tensor(cu, device=dev), max(qlens), kc, vc,
                                bt, torch.as_tensor(lens, device=dev), x["scale"], err,
                                workspace=ws)
        outs.append(out)
    torch.cuda.synchronize()
    assert err.item() == 0
    _same_bits(outs[1], outs[0], "chunked-prefill output")
    ref = oracle.paged_prefill(W.bits(q), cu, W.bits(ks).ravel(), W.bits(vs).ravel(),
                               BS * HKV * d, x["bt"], lens, HKV, BS, x["scale"])
    assert_attention_close(outs[1], ref, "chunked prefill over a pool past 2^31 elements")


def test_scored_append_beyond_2_31_elements():
    """The append that also writes each new token's ||V|| / ||K|| into the paged score
    pool ([KVL] "PagedEviction 块级驱逐机制"): the KV rows and the score entries land
    in the same blocks as in the small pool, bit for bit."""
    dev, d = "cuda", 128
    x = _common(1500, d)
    base, n_big = _layout(BS * HKV * d, x["n_small"])
    g = x["g"]
    ks = torch.randn(x["n_small"], BS, HKV, d, generator=g).to(torch.bfloat16).to(dev)
    vs = torch.randn(x["n_small"], BS, HKV, d, generator=g).to(torch.bfloat16).to(dev)
    ss = torch.rand(x["n_small"], BS, HKV, generator=g).to(dev)
    kb, ids = _place(ks, n_big, base, float("nan"))
    vb, _ = _place(vs, n_big, base, float("nan"))
    sb, _ = _place(ss, n_big, base, float("nan"))
    bt_s = torch.as_tensor(x["bt"], device=dev)
    bt_b = torch.as_tensor(np.where(x["bt"] >= 0, base + STEP * x["bt"], -1).astype(np.int32),
                           device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pk.pa_append_kv_scored(x["k_new"], x["v_new"], ks, vs, ss, bt_s, x["pos"], err)
    pk.pa_append_kv_scored(x["k_new"], x["v_new"], kb, vb, sb, bt_b, x["pos"], err)
    torch.cuda.synchronize()
    assert err.item() == 0
    _same_bits(kb[ids], ks, "K blocks")
    _same_bits(vb[ids], vs, "V blocks")
    _same_bits(sb[ids], ss, "score pool blocks")


def test_prefill_compression_beyond_2_31_elements():
    """PagedEviction's prefill stage ([KVL]): score, keep the budget's highest-ranking
    prompt tokens, and pack them at positions 0.. of each sequence through its block
    table.  Written into a pool past 2^31 elements, the blocks equal the small pool's."""
    dev, d, budget = "cuda", 128, 256
    g = torch.Generator().manual_seed(1600)
    plens = [500, 1500, 40]
    cu = torch.as_tensor(np.concatenate([[0], np.cumsum(plens)]).astype(np.int32), device=dev)
    T = int(cu[-1])
    k = torch.randn(T, HKV, d, generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn(T, HKV, d, generator=g).to(torch.bfloat16).to(dev)
    B, nb = len(plens), budget // BS
    n_small = B * nb + 2
    perm = np.random.default_rng(1600).permutation(n_small).astype(np.int32)
    bt = perm[:B * nb].reshape(B, nb)
    base, n_big = _layout(BS * HKV * d, n_small)
    ks = torch.zeros(n_small, BS, HKV, d, dtype=torch.bfloat16, device=dev)
    vs = torch.zeros_like(ks)
    kb, ids = _place(ks, n_big, base, float("nan"))
    vb, _ = _place(vs, n_big, base, float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    res = []
    for kc, vc, table in ((ks, vs, bt), (kb, vb, base + STEP * bt)):
        scores = torch.empty(T, dtype=torch.float32, device=dev)
        keep = torch.full((B, budget), -7, dtype=torch.int32, device=dev)
        kept = torch.full((B,), -7, dtype=torch.int32, device=dev)
        pk.pe_prefill_compress(kc, vc, torch.as_tensor(table.astype(np.int32), device=dev), k, v,
                               cu, scores, keep, kept, err)
        res.append((keep, kept))
    torch.cuda.synchronize()
    assert err.item() == 0
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
    assert res[0][1].tolist() == [min(n, budget) for n in plens]
    _same_bits(kb[ids], ks, "K blocks after the pack")
    _same_bits(vb[ids], vs, "V blocks after the pack")
