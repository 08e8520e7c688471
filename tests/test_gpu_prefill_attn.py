"""GPU parity of the multi-query (chunked prefill) paged attention through the
C ABI against the fp64 oracle: |err| <= 2e-3 + 1e-2 |ref| on every output of
medium cases (several 64-row query tiles, 64-token K/V tiles, ragged tails,
GQA group sizes 1..16, d 64 and 128, block sizes 12, 16 and 256), the
append-then-attend sequence, mixed chunk + decode batches, invalid lengths,
sampled rows of a full-size 512-token chunk at 8K context, and 16 seeded random
shapes; each in the one-CTA-per-query-tile mode and in the balanced mode
(workspace given: tile ranges cut across SMs, partial results merged), which
bench.py times."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_attention_close
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _case(lens, qlens, Hq, Hkv, d, bs, seed, spare=4):
    g = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    nb = [max(1, -(-int(n) // bs)) for n in lens]
    N = sum(nb) + spare
    perm = rng.permutation(N).astype(np.int32)
    MB = max(nb)
    bt = np.full((len(lens), MB), -1, np.int32)
    c = 0
    for b, m in enumerate(nb):
        bt[b, :m] = perm[c:c + m]
        c += m
    k = torch.randn(N, bs, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(N, bs, Hkv, d, generator=g).to(torch.bfloat16)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = torch.randn(int(cu[-1]), Hq, d, generator=g).to(torch.bfloat16)
    return dict(k=k, v=v, q=q, bt=bt, cu=cu, lens=np.asarray(lens, np.int32), Hq=Hq, Hkv=Hkv,
                d=d, bs=bs, N=N, qlens=list(qlens))


def _workspace(c, balanced):
    """The balanced mode's workspace, filled with 0xff (stale scratch), or None."""
    if not balanced:
        return None
    ws = pk.alloc_prefill_workspace(len(c["lens"]), c["Hq"], c["Hkv"], c["d"], c["bs"],
                                    max(c["qlens"] + [0]), "cuda")
    if ws is not None:
        ws.fill_(0xFF)
    return ws


def _padded(pool, pad):
    """A [N, bs, Hkv, d] view of a device buffer with bs + pad slots per block whose
    extra slots hold NaN (block stride (bs + pad)·Hkv·d), and those extra slots."""
    N, bs, Hkv, d = pool.shape
    big = torch.full((N, bs + pad, Hkv, d), float("nan"), dtype=pool.dtype, device="cuda")
    big[:, :bs].copy_(pool)
    return big[:, :bs], big[:, bs:]


def _run(c, err_expected=0, balanced=False, pad=0):
    dev = "cuda"
    out = torch.full(c["q"].shape, float("nan"), dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    if pad:
        (kd, kgap), (vd, vgap) = _padded(c["k"], pad), _padded(c["v"], pad)
    else:
        kd, vd = c["k"].to(dev), c["v"].to(dev)
    pk.pa_prefill_attention(out, c["q"].to(dev), torch.as_tensor(c["cu"]).to(dev),
                            max(c["qlens"] + [0]), kd, vd,
                            torch.as_tensor(c["bt"]).to(dev), torch.as_tensor(c["lens"]).to(dev),
                            c["d"] ** -0.5, err, workspace=_workspace(c, balanced))
    torch.cuda.synchronize()
    assert err.item() == err_expected
    if pad:
        assert torch.isnan(kgap).all() and torch.isnan(vgap).all()
    return out


def _oracle(c):
    stride = c["bs"] * c["Hkv"] * c["d"]
    return oracle.paged_prefill(W.bits(c["q"]), c["cu"], W.bits(c["k"]).ravel(),
                                W.bits(c["v"]).ravel(), stride, c["bt"], c["lens"], c["Hkv"],
                                c["bs"], c["d"] ** -0.5)


CASES = {
    # Llama-3-8B shape: a 512-token chunk, a whole prompt in one chunk, decodes, an empty row
    "g4d128": ([2048, 700, 37, 5, 1100], [512, 1, 37, 0, 100], 32, 8, 128, 16),
    "g1d128": ([300, 129], [130, 64], 8, 8, 128, 16),
    "g16d128": ([900, 64], [70, 3], 64, 4, 128, 16),
    "g2d64": ([513, 1000, 65], [257, 1, 65], 16, 8, 64, 16),
    "g8d64bs12": ([250, 97], [99, 97], 32, 4, 64, 12),
    "g4bs256": ([1500, 2000], [300, 513], 32, 8, 128, 256),
}


@pytest.mark.parametrize("balanced", [False, True])
@pytest.mark.parametrize("key", list(CASES))
def test_prefill_attention_medium(key, balanced):
    lens, qlens, Hq, Hkv, d, bs = CASES[key]
    c = _case(lens, qlens, Hq, Hkv, d, bs, seed=100 + list(CASES).index(key))
    out = _run(c, balanced=balanced)
    assert_attention_close(out, _oracle(c), key)


@pytest.mark.parametrize("balanced", [False, True])
@pytest.mark.parametrize("key", ["g4d128", "g2d64"])
def test_prefill_attention_padded_block_stride(key, balanced):
    """Pools whose blocks sit (bs + 3)·Hkv·d elements apart, the extra slots holding
    NaN: the kernels follow the block stride and read nothing between blocks."""
    lens, qlens, Hq, Hkv, d, bs = CASES[key]
    c = _case(lens, qlens, Hq, Hkv, d, bs, seed=141 + list(CASES).index(key))
    out = _run(c, balanced=balanced, pad=3)
    assert_attention_close(out, _oracle(c), f"{key}, padded block stride")


@pytest.mark.parametrize("qlens", [[64], [256, 1], [512, 0, 512]])
def test_balanced_mode_with_few_long_items(qlens):
    """Few query tiles over long contexts: every tile range is cut across many SMs
    (one item in many parts), so the merge combines many partial results."""
    lens = [6000 + 37 * b for b in range(len(qlens))]
    c = _case(lens, qlens, 32, 8, 128, 16, seed=21 + len(qlens))
    out = _run(c, balanced=True)
    assert_attention_close(out, _oracle(c), f"balanced, q lens {qlens}")


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def test_balanced_mode_items_a_multiple_of_the_sms():
    """As many items as SMs (one kv head, a group of 8, one 32-token query tile per
    sequence): every item runs whole in the first launch and the range launch has
    no tiles; its CTAs only wait for the first launch."""
    P = _sms()
    rng = np.random.default_rng(51)
    lens = [int(x) for x in rng.integers(33, 400, P)]
    qlens = [int(x) for x in rng.integers(1, 33, P)]
    c = _case(lens, qlens, 8, 1, 128, 16, seed=52)
    assert_attention_close(_run(c, balanced=True), _oracle(c), "items = SMs")


def test_balanced_mode_more_than_two_waves_of_whole_items():
    """2 P + 13 items: two full waves of whole items (the range launch can start only
    after every whole-item CTA has started), then 13 long items cut into many
    one-tile ranges, each merged from several parts."""
    P = _sms()
    rng = np.random.default_rng(53)
    lens = [int(x) for x in rng.integers(33, 300, 2 * P)] + [2500 + 97 * i for i in range(13)]
    qlens = [int(x) for x in rng.integers(1, 33, 2 * P)] + [32] * 13
    c = _case(lens, qlens, 8, 1, 128, 16, seed=54)
    assert_attention_close(_run(c, balanced=True), _oracle(c), "2 P + 13 items")


def test_balanced_mode_is_deterministic():
    c = _case([3000, 800], [512, 300], 32, 8, 128, 16, seed=31)
    a = _run(c, balanced=True)
    b = _run(c, balanced=True)
    assert torch.equal(a, b)


def test_append_chunk_then_attend():
    """The chunk's rows written by pa_append_kv (n_new = chunk) and then
    attended: the same as the oracle's append + prefill attention."""
    Hq, Hkv, d, bs = 32, 8, 128, 16
    old, chunk = np.array([1000, 300], np.int32), [512, 200]
    lens = old + np.array(chunk, np.int32)
    c = _case(lens, chunk, Hq, Hkv, d, bs, seed=9)
    g = torch.Generator().manual_seed(10)
    kn = torch.randn(2, 512, Hkv, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(2, 512, Hkv, d, generator=g).to(torch.bfloat16)
    stride = bs * Hkv * d
    kc, vc = W.bits(c["k"]).ravel().copy(), W.bits(c["v"]).ravel().copy()
    dev = "cuda"
    kd, vd = c["k"].to(dev), c["v"].to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    bt = torch.as_tensor(c["bt"]).to(dev)
    for b in range(2):
        n = chunk[b]
        pk.pa_append_kv(kn[b:b + 1, :n].contiguous().to(dev), vn[b:b + 1, :n].contiguous().to(dev),
                        kd, vd, bt[b:b + 1], torch.as_tensor(old[b:b + 1]).to(dev), err)
        oracle.append_kv(W.bits(kn[b:b + 1, :n]), W.bits(vn[b:b + 1, :n]), kc, vc, stride,
                         c["bt"][b:b + 1], old[b:b + 1], bs)
    out = torch.empty(c["q"].shape, dtype=torch.bfloat16, device=dev)
    pk.pa_prefill_attention(out, c["q"].to(dev), torch.as_tensor(c["cu"]).to(dev), 512, kd, vd,
                            bt, torch.as_tensor(lens).to(dev), d ** -0.5, err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oracle.paged_prefill(W.bits(c["q"]), c["cu"], kc, vc, stride, c["bt"], lens, Hkv, bs,
                               d ** -0.5)
    assert_attention_close(out, ref, "append + prefill attention")


def test_single_query_rows_match_decode_kernel_results():
    """q_len = 1 everywhere: both the prefill kernel and the decode kernel
    within tolerance of the same oracle."""
    lens = [1, 17, 300, 1025]
    c = _case(lens, [1] * 4, 32, 8, 128, 16, seed=11)
    out = _run(c)
    ref = _oracle(c)
    assert_attention_close(out, ref, "prefill kernel, q_len 1")
    stride = 16 * 8 * 128
    ref_dec = oracle.paged_decode(W.bits(c["q"]), W.bits(c["k"]).ravel(), W.bits(c["v"]).ravel(),
                                  stride, c["bt"], c["lens"], 8, 16, 128 ** -0.5)
    assert np.array_equal(ref, ref_dec)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("balanced", [False, True])
def test_invalid_query_length_gives_zero_rows_and_flag(d, balanced):
    c = _case([50, 10], [20, 11], 8, 2, d, 16, seed=12)
    out = _run(c, err_expected=pk.PA_DEV_BAD_LEN, balanced=balanced)
    ref = _oracle(c)
    assert not ref[20:].any()
    assert (out[20:].float() == 0).all()
    assert_attention_close(out[:20], ref[:20], "valid sequence next to an invalid one")


@pytest.mark.parametrize("balanced", [False, True])
def test_full_size_chunk_sampled_rows(balanced):
    """The last 512-token chunk of an 8192-token prompt, Llama-3-8B shape, 4
    sequences: sampled query rows against the decode oracle at the row's own
    position (causality makes query i of the chunk a decode over p + 1 tokens)."""
    Hq, Hkv, d, bs = 32, 8, 128, 16
    lens = [8192] * 4
    c = _case(lens, [512] * 4, Hq, Hkv, d, bs, seed=13)
    out = _run(c, balanced=balanced).cpu()
    rng = np.random.default_rng(14)
    stride = bs * Hkv * d
    kb, vb = W.bits(c["k"]).ravel(), W.bits(c["v"]).ravel()
    for b in range(4):
        rows = np.concatenate([[0, 511], rng.integers(1, 511, 6)])
        for i in rows:
            p = 8192 - 512 + int(i)
            qrow = c["q"][c["cu"][b] + int(i)].unsqueeze(0)
            ref = oracle.paged_decode(W.bits(qrow), kb, vb, stride, c["bt"][b:b + 1],
                                      np.array([p + 1], np.int32), Hkv, bs, d ** -0.5)
            assert_attention_close(out[c["cu"][b] + int(i)].unsqueeze(0), ref, f"seq {b} row {i}")



@pytest.mark.parametrize("balanced", [False, True])
def test_dominant_tokens_keep_the_tolerance(balanced):
    """Rows whose softmax puts almost all weight on two or three tokens with values of
    opposite sign (the case where one rounding of the weights shows most): keys equal
    to a multiple of the query make those tokens dominate."""
    c = _case([900, 400], [128, 64], 32, 8, 128, 16, seed=52)
    k = c["k"].float()
    q = c["q"].float()
    bt = c["bt"]
    for b, (toks, base) in enumerate((([3, 500, 777], 0), ([10, 399], 128))):
        for n, t in enumerate(toks):
            blk, off = bt[b, t // 16], t % 16
            # head 0's query rows of this sequence all see these keys strongly
            k[blk, off, 0] = q[c["cu"][b], 0] * (1.2 + 0.05 * n)
    c["k"] = k.to(torch.bfloat16)
    out = _run(c, balanced=balanced)
    assert_attention_close(out, _oracle(c), "few dominant tokens")


@pytest.mark.parametrize("balanced", [False, True])
def test_late_dominant_tokens_rescale_the_output(balanced):
    """Online softmax across K/V tiles ([KVP] "PagedAttention 的算子"): keys that
    dominate only in later tiles, each stronger than the last, move the rows' running
    maximum by more than a factor 2^8 after O already holds earlier tiles, so the
    kernel rescales O mid-row (the lazy rescale that random N(0, 1) logits never
    reach).  Head 0's rows of each chunk see logits of about 10, 20 and 33 (log2
    units) at those tokens against about 4 elsewhere."""
    c = _case([900, 700], [128, 256], 32, 8, 128, 16, seed=53)
    k = c["k"].float()
    q = c["q"].float()
    bt = c["bt"]
    for b, toks in enumerate(((300, 600, 850), (200, 450, 690))):
        for t, f in zip(toks, (0.6, 1.2, 2.0)):
            blk, off = bt[b, t // 16], t % 16
            k[blk, off, 0] = q[c["cu"][b], 0] * f
    c["k"] = k.to(torch.bfloat16)
    out = _run(c, balanced=balanced)
    assert_attention_close(out, _oracle(c), "late dominant tokens")


def _random_case(i):
    """Seeded random chunked-prefill shape: 1-6 sequences, chunks from 0 rows to the
    whole context, lengths around tile and block boundaries, G 1-16, d 64 / 128,
    block sizes 12, 16, 32 and 256."""
    rng = np.random.default_rng(5000 + i)
    Hkv = int(rng.choice([1, 2, 4, 8]))
    G = int(rng.choice([1, 2, 4, 8, 16]))
    d = int(rng.choice([64, 128, 128]))
    bs = int(rng.choice([12, 16, 16, 32, 256]))
    B = int(rng.integers(1, 7))
    lens, qlens = [], []
    for _ in range(B):
        n = int(rng.choice([1, 63, 64, 65, 127, 128, 129, 255, 256, 257])) \
            if rng.random() < 0.3 else int(rng.integers(1, 2500))
        q = int(rng.choice([0, 1, n, min(n, 64), min(n, 129), min(n, 300)])) \
            if rng.random() < 0.5 else int(rng.integers(0, min(n, 700) + 1))
        lens.append(n)
        qlens.append(q)
    return lens, qlens, G * Hkv, Hkv, d, bs


@pytest.mark.parametrize("balanced", [False, True])
@pytest.mark.parametrize("i", range(16))
def test_prefill_attention_random_shapes(i, balanced):
    lens, qlens, Hq, Hkv, d, bs = _random_case(i)
    c = _case(lens, qlens, Hq, Hkv, d, bs, seed=5000 + i)
    out = _run(c, balanced=balanced)
    assert_attention_close(out, _oracle(c), f"random case {i}: {lens} {qlens} G{Hq // Hkv} "
                                            f"d{d} bs{bs}")
