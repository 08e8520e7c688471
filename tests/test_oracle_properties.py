"""Property-based pins of the fp64 oracle (CPU): random small shapes, block sizes,
GQA groups and ragged lengths (zero included), each checked against an independent
statement of the result: torch's fp64 scaled_dot_product_attention on K/V gathered
with numpy indexing, numpy norms, a brute-force keep set, and a stateful
token -> slot map.  Examples are bounded so the file runs in seconds."""
import math

import numpy as np
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=30, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow])


def bits(x):
    return torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def vals(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@st.composite
def paged_case(draw):
    Hkv = draw(st.sampled_from([1, 2, 4]))
    G = draw(st.sampled_from([1, 2, 4, 8]))
    d = draw(st.sampled_from([4, 8, 16]))
    bs = draw(st.integers(1, 9))
    B = draw(st.integers(1, 4))
    lens = draw(st.lists(st.integers(0, 40), min_size=B, max_size=B))
    spare = draw(st.integers(0, 5))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    rng = np.random.default_rng(seed)
    nb = [-(-n // bs) for n in lens]
    N = sum(nb) + spare + 1
    MB = max(nb + [1])
    perm = rng.permutation(N).astype(np.int32)
    bt = np.full((B, MB), -1, np.int32)
    k = 0
    for b, m in enumerate(nb):
        bt[b, :m] = perm[k:k + m]
        k += m
    kc = bits(rng.standard_normal((N, bs, Hkv, d)))
    vc = bits(rng.standard_normal((N, bs, Hkv, d)) * rng.uniform(0.1, 4))
    q = bits(rng.standard_normal((B, G * Hkv, d)))
    return dict(B=B, Hq=G * Hkv, Hkv=Hkv, d=d, bs=bs, N=N, bt=bt,
                lens=np.asarray(lens, np.int32), kc=kc, vc=vc, q=q)


def gathered(c, b):
    n = int(c["lens"][b])
    ids = c["bt"][b, : -(-n // c["bs"])]
    K = vals(c["kc"][ids]).reshape(-1, c["Hkv"], c["d"])[:n]
    V = vals(c["vc"][ids]).reshape(-1, c["Hkv"], c["d"])[:n]
    return K, V


@SETTINGS
@given(paged_case())
def test_decode_is_sdpa_over_the_gathered_context(c):
    Hq, Hkv, d = c["Hq"], c["Hkv"], c["d"]
    out = oracle.paged_decode(c["q"], c["kc"].ravel(), c["vc"].ravel(), c["bs"] * Hkv * d,
                              c["bt"], c["lens"], Hkv, c["bs"], 1 / math.sqrt(d))
    q = vals(c["q"])
    for b in range(c["B"]):
        if c["lens"][b] == 0:
            assert not out[b].any()
            continue
        K, V = gathered(c, b)
        Kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
        Vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b]).unsqueeze(1), Kt, Vt, scale=1 / math.sqrt(d))[:, 0].numpy()
        np.testing.assert_allclose(out[b], ref, rtol=1e-11, atol=1e-12)


@SETTINGS
@given(paged_case(), st.integers(1, 6))
def test_chunked_prefill_is_causal_sdpa(c, qmax):
    Hq, Hkv, d = c["Hq"], c["Hkv"], c["d"]
    rng = np.random.default_rng(int(c["lens"].sum()) + qmax)
    qlens = [int(rng.integers(0, min(qmax, n) + 1)) for n in c["lens"]]
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    qp = bits(rng.standard_normal((int(cu[-1]), Hq, d)))
    out = oracle.paged_prefill(qp, cu, c["kc"].ravel(), c["vc"].ravel(), c["bs"] * Hkv * d,
                               c["bt"], c["lens"], Hkv, c["bs"], 1 / math.sqrt(d))
    for b, ql in enumerate(qlens):
        if ql == 0:
            continue
        n = int(c["lens"][b])
        K, V = gathered(c, b)
        Kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
        Vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
        qt = torch.from_numpy(vals(qp[cu[b]:cu[b + 1]])).permute(1, 0, 2)
        allowed = torch.arange(n)[None, :] <= (n - ql + torch.arange(ql))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=allowed,
                                                               scale=1 / math.sqrt(d))
        np.testing.assert_allclose(out[cu[b]:cu[b + 1]], ref.permute(1, 0, 2).numpy(),
                                   rtol=1e-11, atol=1e-12)


@SETTINGS
@given(paged_case())
def test_scores_and_block_choice_from_numpy(c):
    Hkv, d, bs = c["Hkv"], c["d"], c["bs"]
    s = oracle.score_tokens(c["kc"].ravel(), c["vc"].ravel(), bs * Hkv * d, c["bt"], c["lens"],
                            Hkv, d, bs)
    ev, means, _ = oracle.select_evict_block(s, c["lens"], bs)
    for b in range(c["B"]):
        n = int(c["lens"][b])
        K, V = gathered(c, b)
        np.testing.assert_allclose(s[b, :n], np.linalg.norm(V, axis=-1) /
                                   np.linalg.norm(K, axis=-1), rtol=1e-13)
        full = n // bs
        m = [s[b, j * bs:(j + 1) * bs].mean() for j in range(full)]
        assert ev[b] == (int(np.argmin(m)) if full else -1)   # argmin: first of equal minima
        np.testing.assert_allclose(means[b, :full], m, rtol=1e-13)


@SETTINGS
@given(st.lists(st.integers(0, 12), min_size=1, max_size=4), st.integers(1, 8),
       st.integers(0, 2 ** 31 - 1))
def test_prefill_keep_set_is_the_brute_force_best(lens, budget, seed):
    """The kept tokens are the `budget` best by (score, later index) with NaN lowest:
    checked against a sort of Python tuples."""
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    scores = rng.choice([0.5, 1.0, 2.0, np.inf, np.nan, -0.0, 0.0], size=int(cu[-1]))
    keep, kept = oracle.prefill_select(scores, cu, budget)
    for b, n in enumerate(lens):
        x = scores[cu[b]:cu[b + 1]]
        key = [(-np.inf if np.isnan(v) else v, i) for i, v in enumerate(x)]
        want = sorted(i for _, i in sorted(key, reverse=True)[:min(n, budget)])
        assert kept[b] == min(n, budget)
        assert keep[b, :kept[b]].tolist() == want
        assert (keep[b, kept[b]:] == -1).all()


@SETTINGS
@given(paged_case(), st.integers(0, 2 ** 31 - 1))
def test_compaction_keeps_every_surviving_token_at_its_slot(c, seed):
    """Any set of marked blocks: the surviving tokens keep their slots (at positions
    shifted down by bs per evicted full block before them), partial blocks never go."""
    rng = np.random.default_rng(seed)
    bs, B = c["bs"], c["B"]
    MB = c["bt"].shape[1]
    mask = (rng.random((B, MB)) < 0.4).astype(np.uint8)
    nbt, nlen, fr = oracle.evict_compact_mask(c["bt"], c["lens"], mask, bs)
    for b in range(B):
        n = int(c["lens"][b])
        gone = [j for j in range(n // bs) if mask[b, j]]
        assert nlen[b] == n - bs * len(gone)
        assert fr[b, :len(gone)].tolist() == [int(c["bt"][b, j]) for j in gone]
        for p in range(n):
            j = p // bs
            if j in gone:
                continue
            q = p - bs * sum(1 for g in gone if g < j)
            assert oracle.slot(nbt[b], q, bs) == oracle.slot(c["bt"][b], p, bs)


@SETTINGS
@given(st.integers(1, 6), st.sampled_from([4, 16, 64]), st.floats(-20, 20),
       st.integers(0, 2 ** 31 - 1))
def test_int8_quantiser_bounds(rows, d, log2_mag, seed):
    """Codes in [-127, 127] with the row's amax at +-127, scale = amax / 127 in fp32, and
    |scale * code - x| <= scale / 2 plus the one fp32 rounding of x / scale; an all-zero
    row gets scale 0 and codes 0."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, d)) * 2.0 ** log2_mag
    x[0] = 0.0
    b = bits(x)
    codes, scales = oracle.quantize_int8(b)
    xv = vals(b)
    amax = np.abs(xv).max(axis=1)
    assert np.array_equal(scales, (amax.astype(np.float32) / np.float32(127)).astype(np.float32))
    assert scales[0] == 0 and not codes[0].any()
    nz = amax > 0
    assert (np.abs(codes[nz]).max(axis=1) == 127).all() and np.abs(codes).max() <= 127
    s = scales[:, None].astype(np.float64)
    assert (np.abs(s * codes - xv) <= s * (0.5 + 127 * 2.0 ** -24)).all()


@SETTINGS
@given(st.floats(-12, 8.7), st.integers(0, 2 ** 31 - 1))
def test_e4m3_cast_is_torchs_in_range_and_saturates_beyond(log2_mag, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(256) * 2.0 ** log2_mag
    b = bits(x)
    xv = vals(b)
    codes = oracle.quantize_e4m3(b)
    ok = np.abs(xv) <= 448.0
    ref = torch.as_tensor(xv[ok].astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8)
    assert np.array_equal(codes[ok], ref.numpy())
    big = ~ok
    assert np.array_equal(codes[big], np.where(xv[big] > 0, 0x7e, 0xfe).astype(np.uint8))


def _sdpa_rows(q, K, V, G, d):
    Kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(G, 0)
    Vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(G, 0)
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).unsqueeze(1), Kt, Vt, scale=1 / math.sqrt(d))[:, 0].numpy()


@SETTINGS
@given(paged_case(), st.sampled_from(["int8", "fp8"]))
def test_quantised_decode_is_sdpa_on_the_stored_values(c, kind):
    """INT8: the values are scale * code per (token, head) row; FP8: each e4m3 code's
    exact value.  Either way the decode equals fp64 SDPA on those values."""
    Hq, Hkv, d, bs = c["Hq"], c["Hkv"], c["d"], c["bs"]
    stride = bs * Hkv * d
    if kind == "int8":
        kq, ks = oracle.quantize_int8(c["kc"])
        vq, vs = oracle.quantize_int8(c["vc"])
        out = oracle.paged_decode_int8(c["q"], kq.ravel(), vq.ravel(), ks.ravel(), vs.ravel(),
                                       stride, c["bt"], c["lens"], Hkv, bs, 1 / math.sqrt(d))
        kd = ks[..., None].astype(np.float64) * kq
        vd = vs[..., None].astype(np.float64) * vq
    else:
        k8, v8 = oracle.quantize_e4m3(c["kc"]), oracle.quantize_e4m3(c["vc"])
        out = oracle.paged_decode_fp8(c["q"], k8.ravel(), v8.ravel(), stride, c["bt"],
                                      c["lens"], Hkv, bs, 1 / math.sqrt(d))
        kd, vd = oracle.e4m3_values(k8), oracle.e4m3_values(v8)
    q = vals(c["q"])
    for b in range(c["B"]):
        n = int(c["lens"][b])
        if n == 0:
            assert not out[b].any()
            continue
        ids = c["bt"][b, : -(-n // bs)]
        K = kd[ids].reshape(-1, Hkv, d)[:n]
        V = vd[ids].reshape(-1, Hkv, d)[:n]
        np.testing.assert_allclose(out[b], _sdpa_rows(q[b], K, V, Hq // Hkv, d), rtol=1e-11,
                                   atol=1e-12)
