"""Pins of the fp64 oracle against what the pages and the mathematics fix.

CPU only.  None of these re-types the oracle's own code: each checks a printed
value, a closed form, an invariant, a special case that reduces to a textbook
or library routine, or a brute-force/stateful restatement on tiny inputs.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_396_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(x) -> np.ndarray:
    return torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def bf16_vals(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rand_case(seed, B=3, Hq=8, Hkv=2, d=16, bs=4, N=40, lens=(1, 7, 13)):
    rng = np.random.default_rng(seed)
    perm = rng.permutation(N).astype(np.int32)
    MB = max(-(-n // bs) for n in lens)
    bt = np.full((B, MB), -1, np.int32)
    k = 0
    for b, n in enumerate(lens):
        for j in range(-(-n // bs)):
            bt[b, j] = perm[k]
            k += 1
    kc = bf16_bits(rng.standard_normal((N, bs, Hkv, d)))
    vc = bf16_bits(rng.standard_normal((N, bs, Hkv, d)))
    q = bf16_bits(rng.standard_normal((B, Hq, d)))
    return dict(q=q, kc=kc, vc=vc, bt=bt, lens=np.asarray(lens, np.int32), B=B, Hq=Hq, Hkv=Hkv,
                d=d, bs=bs, N=N)


def run_decode(c, scale=None):
    scale = 1.0 / math.sqrt(c["d"]) if scale is None else scale
    return oracle.paged_decode(c["q"], c["kc"].ravel(), c["vc"].ravel(),
                               c["bs"] * c["Hkv"] * c["d"], c["bt"], c["lens"], c["Hkv"],
                               c["bs"], scale)


def gather_logical(c, b):
    """K, V of sequence b in logical order via plain numpy indexing of the table."""
    n = int(c["lens"][b])
    ids = c["bt"][b, : -(-n // c["bs"])]
    K = bf16_vals(c["kc"][ids]).reshape(-1, c["Hkv"], c["d"])[:n]
    V = bf16_vals(c["vc"][ids]).reshape(-1, c["Hkv"], c["d"])[:n]
    return K, V


# ------------------------------------------------------------------ sizes
def _golden_sizes():
    rows = []
    with open(os.path.join(GOLDEN, "kv_sizes.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append(line.split())
    return rows


def test_kv_bytes_per_token_printed_values():
    rows = _golden_sizes()
    seen = set()
    for kind, name, L, nkv, d, elt, *vals in rows:
        L, nkv, d, elt = int(L), int(nkv), int(d), int(elt)
        per_tok = oracle.kv_bytes_per_token(L, nkv, d, elt)
        if kind == "token":
            assert per_tok == int(vals[0])
        elif kind == "context":
            for item in vals:
                ctx, nbytes = map(int, item.split(":"))
                assert per_tok * ctx == nbytes
        elif kind == "half":       # the page's 160 KB is K alone (or V alone)
            assert per_tok // 2 == int(vals[0]) and per_tok == 2 * int(vals[0])
        elif kind == "halfctx":
            ctx, nbytes = map(int, vals[0].split(":"))
            assert per_tok // 2 * ctx == nbytes
        elif kind == "requests":
            ctx, nreq, nbytes = map(int, vals[0].split(":"))
            assert per_tok // 2 * ctx * nreq == nbytes
        seen.add(kind)
    assert seen == {"token", "context", "half", "halfctx", "requests"}


def test_num_blocks_is_ceiling():
    for bs in (1, 2, 7, 16, 256):
        for n in range(0, 600, 3):
            # brute force: smallest k with k*bs >= n
            k = 0
            while k * bs < n:
                k += 1
            assert oracle.num_blocks(n, bs) == k
    # the tiny workload: 38 -> 3 and 101 -> 7 blocks of 16
    assert oracle.num_blocks(38, 16) == 3 and oracle.num_blocks(101, 16) == 7


def test_workload_tables_hold_exactly_the_needed_blocks():
    for key in ("c1", "c2", "c4"):
        cfg = W.CONFIGS[key]
        rng = np.random.default_rng(cfg.seed)
        old = W._old_lens(cfg, rng)
        ctx = old + (1 if cfg.append else 0)
        bt, N = W._allocate(ctx, cfg.block_size, cfg.spare, cfg.pool_blocks, rng)
        used = bt[bt >= 0]
        assert len(np.unique(used)) == len(used) and used.max() < N
        for b in range(cfg.batch):
            assert (bt[b] >= 0).sum() == oracle.num_blocks(int(ctx[b]), cfg.block_size)
    c1 = W.CONFIGS["c1"]
    rng = np.random.default_rng(c1.seed)
    old = W._old_lens(c1, rng)
    bt, N = W._allocate(old + 1, c1.block_size, c1.spare, c1.pool_blocks, rng)
    assert N == 64 and (bt >= 0).sum() == 10


# ------------------------------------------------------------------ slots / append
class BlockTableSim:
    """Stateful restatement of the BlockTable of the vLLM notes (ybb.press §2.1):
    append_slot returns last_block*bs + used slots while the last block has room,
    else takes a new block from the free list and returns its first slot."""

    def __init__(self, bs, free):
        self.bs, self.free, self.table, self.n = bs, list(free), [], 0

    def append_slot(self):
        if self.n % self.bs == 0:            # no block yet, or the last block is full
            self.table.append(self.free.pop())
            s = self.table[-1] * self.bs
        else:
            s = self.table[-1] * self.bs + (self.n % self.bs)
        self.n += 1
        return s


def test_slot_formula_matches_stateful_block_table():
    rng = np.random.default_rng(7)
    for bs in (1, 4, 16, 256):
        sim = BlockTableSim(bs, rng.permutation(200).tolist())
        slots = [sim.append_slot() for _ in range(min(40 * bs, 2000))]
        row = np.asarray(sim.table, np.int32)
        for pos, s in enumerate(slots):
            assert oracle.slot(row, pos, bs) == s
        assert len(set(slots)) == len(slots)


def test_append_then_logical_gather_is_identity():
    rng = np.random.default_rng(11)
    B, Hkv, d, bs, N = 3, 2, 8, 4, 30
    lens = np.array([5, 9, 12], np.int32)
    perm = rng.permutation(N).astype(np.int32)
    MB = 3
    bt = np.full((B, MB), -1, np.int32)
    k = 0
    for b in range(B):
        for j in range(-(-int(lens[b]) // bs)):
            bt[b, j] = perm[k]
            k += 1
    kc = np.zeros(N * bs * Hkv * d, np.uint16)
    vc = np.zeros_like(kc)
    maxlen = int(lens.max())
    kn = bf16_bits(rng.standard_normal((B, maxlen, Hkv, d)))
    vn = bf16_bits(rng.standard_normal((B, maxlen, Hkv, d)))
    # write every token one at a time (decode-style appends)
    for pos in range(maxlen):
        live = [b for b in range(B) if pos < lens[b]]
        oracle.append_kv(kn[live, pos:pos + 1], vn[live, pos:pos + 1], kc, vc, bs * Hkv * d,
                         bt[live], np.full(len(live), pos, np.int32), bs)
    c = dict(kc=kc.reshape(N, bs, Hkv, d), vc=vc.reshape(N, bs, Hkv, d), bt=bt, lens=lens,
             Hkv=Hkv, d=d, bs=bs)
    for b in range(B):
        K, V = gather_logical(c, b)
        n = int(lens[b])
        assert np.array_equal(K, bf16_vals(kn[b, :n]))
        assert np.array_equal(V, bf16_vals(vn[b, :n]))
    # a multi-token append (prefill-style) writes the same pools
    kc2 = np.zeros_like(kc)
    vc2 = np.zeros_like(vc)
    for b in range(B):
        n = int(lens[b])
        oracle.append_kv(kn[b:b + 1, :n], vn[b:b + 1, :n], kc2, vc2, bs * Hkv * d, bt[b:b + 1],
                         np.zeros(1, np.int32), bs)
    assert np.array_equal(kc, kc2) and np.array_equal(vc, vc2)


# ------------------------------------------------------------------ attention
def sdpa_reference(c):
    """Contiguous attention through torch's scaled_dot_product_attention in fp64,
    on the K/V gathered in logical order (an independent library routine)."""
    B, Hq, Hkv, d = c["B"], c["Hq"], c["Hkv"], c["d"]
    out = np.zeros((B, Hq, d))
    q = bf16_vals(c["q"]).reshape(B, Hq, d)
    for b in range(B):
        K, V = gather_logical(c, b)
        Kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)  # [Hq, n, d]
        Vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
        qt = torch.from_numpy(q[b]).unsqueeze(1)  # [Hq, 1, d]
        o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=1 / math.sqrt(d))
        out[b] = o[:, 0].numpy()
    return out


@pytest.mark.parametrize("seed,Hq,Hkv,d,bs", [(1, 8, 2, 16, 4), (2, 4, 4, 8, 3), (3, 16, 2, 64, 16),
                                              (4, 8, 1, 32, 5)])
def test_decode_equals_contiguous_sdpa(seed, Hq, Hkv, d, bs):
    c = rand_case(seed, Hq=Hq, Hkv=Hkv, d=d, bs=bs, N=60, lens=(1, 9, 2 * bs + 1))
    np.testing.assert_allclose(run_decode(c), sdpa_reference(c), rtol=1e-12, atol=1e-12)


def test_decode_invariant_under_physical_block_permutation():
    c = rand_case(5, lens=(3, 11, 17), N=30)
    base = run_decode(c)
    rng = np.random.default_rng(0)
    perm = rng.permutation(c["N"])              # new position of each old block
    inv = np.argsort(perm)
    c2 = dict(c)
    c2["kc"] = c["kc"][inv]                    # block p moves to perm[p]
    c2["vc"] = c["vc"][inv]
    c2["bt"] = np.where(c["bt"] >= 0, perm[np.maximum(c["bt"], 0)], -1).astype(np.int32)
    assert np.array_equal(run_decode(c2), base)


def test_decode_len_one_returns_v0_and_len_zero_returns_zero():
    c = rand_case(6, lens=(1, 1, 0))
    out = run_decode(c)
    for b in range(2):
        _, V = gather_logical(c, b)
        for i in range(c["Hq"]):
            assert np.array_equal(out[b, i], V[0, i // (c["Hq"] // c["Hkv"])])
    assert not out[2].any()


def test_decode_equal_keys_gives_mean_of_values():
    c = rand_case(7, lens=(5, 13, 8))
    kc = c["kc"].copy()
    kc[...] = bf16_bits(np.linspace(-1, 1, c["d"]))  # every key the same vector
    c["kc"] = kc
    out = run_decode(c)
    for b in range(c["B"]):
        _, V = gather_logical(c, b)
        G = c["Hq"] // c["Hkv"]
        for i in range(c["Hq"]):
            np.testing.assert_allclose(out[b, i], V[:, i // G].mean(0), rtol=1e-13, atol=1e-13)


def test_decode_gqa_groups_are_contiguous():
    # V[t, h, :] = h + 1 everywhere: each output is the constant of its kv head,
    # so query head i must read kv head i // G (not i % Hkv).
    c = rand_case(8, Hq=8, Hkv=4, lens=(6, 3, 10))
    vc = np.empty_like(c["vc"])
    for h in range(4):
        vc[:, :, h, :] = bf16_bits(np.full(c["d"], h + 1.0))
    c["vc"] = vc
    out = run_decode(c)
    for i in range(8):
        np.testing.assert_allclose(out[:, i, :], i // 2 + 1.0, rtol=0, atol=1e-14)


def test_decode_dominant_key_selects_its_value():
    c = rand_case(9, Hq=2, Hkv=1, lens=(12, 12, 12))
    kc = c["kc"].copy()
    qv = bf16_vals(c["q"])
    for b in range(c["B"]):
        t = 5 + b
        blk, off = c["bt"][b, t // c["bs"]], t % c["bs"]
        kc[blk, off, 0] = bf16_bits(qv[b, 0] * 64.0)   # key aligned with query head 0, huge
    c["kc"] = kc
    out = run_decode(c)
    for b in range(c["B"]):
        _, V = gather_logical(c, b)
        np.testing.assert_allclose(out[b, 0], V[5 + b, 0], atol=1e-8)


def test_decode_never_reads_slots_beyond_len():
    c = rand_case(10, lens=(5, 9, 3))
    base = run_decode(c)
    kc, vc = c["kc"].copy(), c["vc"].copy()
    nan = bf16_bits(np.full(c["d"], np.nan))
    for b in range(c["B"]):
        n = int(c["lens"][b])
        last = c["bt"][b, (n - 1) // c["bs"]]
        for off in range(n % c["bs"] or c["bs"], c["bs"]):
            kc[last, off] = nan
            vc[last, off] = nan
    c["kc"], c["vc"] = kc, vc
    assert np.array_equal(run_decode(c), base)


def test_decode_brute_force_python_loops_tiny_workload():
    wl = W.generate(W.CONFIGS["c1"], "cpu")
    s = W.compact(wl, 0, range(2))
    kc, vc = s["k_pool"].copy(), s["v_pool"].copy()
    Hkv, d, bs = 2, 64, 16
    oracle.append_kv(s["k_new"], s["v_new"], kc, vc, bs * Hkv * d, s["block_tables"],
                     s["positions"], bs)
    out = oracle.paged_decode(s["q"], kc, vc, bs * Hkv * d, s["block_tables"], s["ctx_lens"],
                              Hkv, bs, 1 / 8)
    qv = bf16_vals(s["q"])
    Kp, Vp = bf16_vals(kc), bf16_vals(vc)
    for b in range(2):
        n = int(s["ctx_lens"][b])
        for i in range(4):
            h = i // 2
            sc = []
            for t in range(n):
                blk = int(s["block_tables"][b][t // bs])
                kv = Kp[blk, t % bs, h]
                sc.append(sum(qv[b, i, e] * kv[e] for e in range(d)) / 8)
            mx = max(sc)
            w = [math.exp(x - mx) for x in sc]
            z = sum(w)
            for e in range(0, d, 9):
                o = sum(w[t] * Vp[int(s["block_tables"][b][t // bs]), t % bs, h, e]
                        for t in range(n)) / z
                assert abs(o - out[b, i, e]) < 1e-12


def test_global_softmax_differs_from_per_block_normalisation():
    """Reading check: the vLLM notes' pseudocode normalises inside each block and
    sums block outputs; the operator of the knowledge page takes softmax over all
    blocks.  The two disagree on any multi-block context, so the oracle must match
    only the global one (already pinned against SDPA)."""
    c = rand_case(12, lens=(9, 9, 9))
    out = run_decode(c)
    b, i = 0, 0
    K, V = gather_logical(c, b)
    q = bf16_vals(c["q"])[b, i]
    per_block = np.zeros(c["d"])
    for j in range(0, 9, c["bs"]):
        s = K[j:j + c["bs"], 0] @ q / math.sqrt(c["d"])
        p = np.exp(s - s.max())
        per_block += (p / p.sum()) @ V[j:j + c["bs"], 0]
    assert np.abs(per_block - out[b, i]).max() > 1e-3



def _pad_blocks(pool, pad, fill):
    """Copy [N, bs, Hkv, d] into [N, bs + pad, Hkv, d] with `fill` in the pad rows and
    return the flat buffer and its block stride."""
    N, bs, Hkv, d = pool.shape
    big = np.full((N, bs + pad, Hkv, d), fill, pool.dtype)
    big[:, :bs] = pool
    return big.ravel(), (bs + pad) * Hkv * d


def test_block_stride_larger_than_a_block_reads_only_the_block():
    """A pool whose blocks sit block_stride > bs*Hkv*d elements apart (the rest of each
    block's span holds NaN, or code 127 / e4m3 NaN for the one-byte pools) gives the
    same decode, chunked-prefill, score and INT8/FP8 results, bit for bit, as the dense
    pool; so the stride is honoured and the padding is never read."""
    c = rand_case(41, Hq=8, Hkv=2, d=16, bs=4, N=20, lens=(5, 13, 8))
    bs, Hkv, d = c["bs"], c["Hkv"], c["d"]
    dense = bs * Hkv * d
    sc = 1 / math.sqrt(d)
    nan16 = np.uint16(0x7fc0)
    kp, stride = _pad_blocks(c["kc"], 3, nan16)
    vp, _ = _pad_blocks(c["vc"], 3, nan16)
    assert stride > dense
    args = (c["bt"], c["lens"], Hkv, bs, sc)
    assert np.array_equal(oracle.paged_decode(c["q"], kp, vp, stride, *args), run_decode(c))
    s_pad = oracle.score_tokens(kp, vp, stride, c["bt"], c["lens"], Hkv, d, bs)
    s_den = oracle.score_tokens(c["kc"].ravel(), c["vc"].ravel(), dense, c["bt"], c["lens"], Hkv,
                                d, bs)
    assert np.array_equal(s_pad, s_den, equal_nan=True)
    cu = np.array([0, 2, 3, 7], np.int32)
    qp = bf16_bits(np.random.default_rng(42).standard_normal((7, c["Hq"], d)))
    assert np.array_equal(oracle.paged_prefill(qp, cu, kp, vp, stride, *args),
                          oracle.paged_prefill(qp, cu, c["kc"].ravel(), c["vc"].ravel(), dense,
                                               *args))
    kq, ks = oracle.quantize_int8(c["kc"])
    vq, vs = oracle.quantize_int8(c["vc"])
    kqp, _ = _pad_blocks(kq, 3, np.int8(127))
    vqp, _ = _pad_blocks(vq, 3, np.int8(127))
    assert np.array_equal(
        oracle.paged_decode_int8(c["q"], kqp, vqp, ks.ravel(), vs.ravel(), stride, *args),
        oracle.paged_decode_int8(c["q"], kq.ravel(), vq.ravel(), ks.ravel(), vs.ravel(), dense,
                                 *args))
    assert np.array_equal(
        oracle.score_tokens_int8(kqp, vqp, ks.ravel(), vs.ravel(), stride, c["bt"], c["lens"],
                                 Hkv, d, bs),
        oracle.score_tokens_int8(kq.ravel(), vq.ravel(), ks.ravel(), vs.ravel(), dense, c["bt"],
                                 c["lens"], Hkv, d, bs), equal_nan=True)
    k8, v8 = oracle.quantize_e4m3(c["kc"]), oracle.quantize_e4m3(c["vc"])
    k8p, _ = _pad_blocks(k8, 3, np.uint8(0x7f))
    v8p, _ = _pad_blocks(v8, 3, np.uint8(0x7f))
    assert np.array_equal(oracle.paged_decode_fp8(c["q"], k8p, v8p, stride, *args),
                          oracle.paged_decode_fp8(c["q"], k8.ravel(), v8.ravel(), dense, *args))


def test_append_with_padded_block_stride_leaves_the_padding():
    """Appending through a padded block stride writes the same block contents as the
    dense append (bf16 and FP8) and leaves every pad element as it was."""
    rng = np.random.default_rng(43)
    B, Hkv, d, bs, N, pad = 2, 2, 8, 4, 10, 2
    bt = np.array([[3, 7, -1], [1, 0, 9]], np.int32)
    kn = bf16_bits(rng.standard_normal((B, 3, Hkv, d)))
    vn = bf16_bits(rng.standard_normal((B, 3, Hkv, d)))
    pos = np.array([2, 7], np.int32)
    for fn, dt, fill in ((oracle.append_kv, np.uint16, 0x7fc0),
                         (oracle.append_kv_fp8, np.uint8, 0x7f)):
        kd = np.full((N, bs, Hkv, d), fill, dt)
        vd = np.full_like(kd, fill)
        fn(kn, vn, kd.reshape(-1), vd.reshape(-1), bs * Hkv * d, bt, pos, bs)
        kp = np.full((N, bs + pad, Hkv, d), fill, dt)
        vp = np.full_like(kp, fill)
        fn(kn, vn, kp.reshape(-1), vp.reshape(-1), (bs + pad) * Hkv * d, bt, pos, bs)
        assert (kp[:, bs:] == fill).all() and (vp[:, bs:] == fill).all()
        assert np.array_equal(kp[:, :bs], kd) and np.array_equal(vp[:, :bs], vd)
        assert (kd != fill).any()
    # INT8: the code pools are padded, the scale pools keep their [N][bs][Hkv] layout
    pools = {}
    for p_ in (0, pad):
        kq = np.full((N, bs + p_, Hkv, d), 127, np.int8)
        vq = np.full_like(kq, 127)
        ks = np.full((N, bs, Hkv), -1, np.float32)
        vs = np.full_like(ks, -1)
        oracle.append_kv_int8(kn, vn, kq.reshape(-1), vq.reshape(-1), ks.reshape(-1),
                              vs.reshape(-1), (bs + p_) * Hkv * d, bt, pos, bs)
        pools[p_] = (kq, vq, ks, vs)
    kq, vq, ks, vs = pools[pad]
    assert (kq[:, bs:] == 127).all() and (vq[:, bs:] == 127).all()
    assert np.array_equal(kq[:, :bs], pools[0][0]) and np.array_equal(vq[:, :bs], pools[0][1])
    assert np.array_equal(ks, pools[0][2]) and np.array_equal(vs, pools[0][3])
    assert (pools[0][0] != 127).any()


def test_prefill_pack_with_padded_block_stride_leaves_the_padding():
    """Packing kept prompt rows through a padded block stride writes the same block
    contents as the dense pack and leaves every pad element as it was."""
    rng = np.random.default_rng(44)
    Hkv, d, bs, N, pad = 2, 8, 4, 12, 3
    cu = np.array([0, 9, 20], np.int32)
    k = bf16_bits(rng.standard_normal((20, Hkv, d)))
    v = bf16_bits(rng.standard_normal((20, Hkv, d)))
    keep, kept = oracle.prefill_select(rng.standard_normal(20), cu, 6)
    bt = np.array([[5, 2], [0, 11]], np.int32)
    out = {}
    for p_ in (0, pad):
        kc = np.full((N, bs + p_, Hkv, d), 0x7fc0, np.uint16)
        vc = np.full_like(kc, 0x7fc0)
        oracle.prefill_pack(k, v, cu, keep, kept, kc.reshape(-1), vc.reshape(-1),
                            (bs + p_) * Hkv * d, bt, bs)
        out[p_] = (kc, vc)
    kc, vc = out[pad]
    assert (kc[:, bs:] == 0x7fc0).all() and (vc[:, bs:] == 0x7fc0).all()
    assert np.array_equal(kc[:, :bs], out[0][0]) and np.array_equal(vc[:, :bs], out[0][1])
    assert (out[0][0] != 0x7fc0).sum() == 12 * Hkv * d


# ------------------------------------------------------------------ scores / eviction
def test_score_is_norm_ratio_closed_forms():
    B, Hkv, d, bs, N = 1, 2, 4, 2, 3
    kc = np.zeros((N, bs, Hkv, d), np.float32)
    vc = np.zeros_like(kc)
    bt = np.array([[2, 0]], np.int32)
    kc[2, 0, 0] = [3, 0, 0, 0]; vc[2, 0, 0] = [0, 4, 0, 0]     # 4/3
    kc[2, 0, 1] = [1, 1, 1, 1]; vc[2, 0, 1] = [2, 2, 2, 2]     # 2
    kc[2, 1, 0] = [0, 0, 0, 0]; vc[2, 1, 0] = [1, 0, 0, 0]     # ||K||=0, ||V||>0: +inf
    kc[2, 1, 1] = [0, 0, 0, 0]; vc[2, 1, 1] = [0, 0, 0, 0]     # both zero: 0
    kc[0, 0, 0] = [1, 2, 2, 0]; vc[0, 0, 0] = [6, 0, 0, 0]     # 6/3
    kc[0, 0, 1] = [-2, 0, 0, 0]; vc[0, 0, 1] = [-0.5, 0, 0, 0]  # 0.25
    s = oracle.score_tokens(bf16_bits(kc).ravel(), bf16_bits(vc).ravel(), bs * Hkv * d, bt,
                            np.array([3], np.int32), Hkv, d, bs)
    assert s.shape == (1, 4, 2)
    np.testing.assert_allclose(s[0, :3].ravel(), [4 / 3, 2, np.inf, 0, 2, 0.25], rtol=1e-15)
    assert np.isnan(s[0, 3]).all()


def test_score_value_proportional_to_key_gives_constant():
    c = rand_case(13, lens=(7, 11, 4), d=32)
    kv = bf16_vals(c["kc"])
    for cval in (0.5, -2.0, 4.0):                       # powers of two: V stays exact in bf16
        vc = bf16_bits(kv * cval)
        s = oracle.score_tokens(c["kc"].ravel(), vc.ravel(), c["bs"] * c["Hkv"] * c["d"], c["bt"],
                                c["lens"], c["Hkv"], c["d"], c["bs"])
        for b in range(c["B"]):
            np.testing.assert_allclose(s[b, :c["lens"][b]], abs(cval), rtol=1e-14)


def test_score_matches_numpy_norms():
    c = rand_case(14, lens=(7, 11, 13), d=16)
    s = oracle.score_tokens(c["kc"].ravel(), c["vc"].ravel(), c["bs"] * c["Hkv"] * c["d"],
                            c["bt"], c["lens"], c["Hkv"], c["d"], c["bs"])
    for b in range(c["B"]):
        K, V = gather_logical(c, b)
        ref = np.linalg.norm(V, axis=-1) / np.linalg.norm(K, axis=-1)
        np.testing.assert_allclose(s[b, :c["lens"][b]], ref, rtol=1e-13)


def test_evict_planted_low_block_and_rules():
    B, Hkv, bs, MB = 4, 2, 4, 5
    rng = np.random.default_rng(3)
    scores = rng.uniform(1.0, 2.0, (B, MB * bs, Hkv))
    lens = np.array([20, 13, 3, 17], np.int32)   # full blocks: 5, 3, 0, 4
    scores[0, 8:12] = 0.5                        # block 2 of seq 0
    scores[1, 4:8] = 0.75                        # block 1 of seq 1
    scores[1, 12:16] = 0.01                      # seq 1 block 3 is partial: not a candidate
    scores[3, :] = 1.5                           # seq 3: all equal -> lowest index wins
    ev, means, gap = oracle.select_evict_block(scores, lens, bs)
    assert ev.tolist() == [2, 1, -1, 0]
    np.testing.assert_allclose(means[0, 2], 0.5)
    assert np.isnan(means[1, 3]) and np.isnan(means[2]).all()
    assert gap[3] == 0.0 and gap[2] == np.inf
    # brute force of the block means for seq 0
    for j in range(5):
        assert abs(means[0, j] - scores[0, j * bs:(j + 1) * bs].mean()) < 1e-15
    # gap: second-lowest minus lowest candidate mean, +inf with fewer than two
    for b in range(B):
        m = np.sort(means[b][~np.isnan(means[b])])
        assert gap[b] == (m[1] - m[0] if m.size >= 2 else np.inf)
        assert gap[b] >= 0
    assert gap[0] == np.sort(means[0])[1] - 0.5 > 0.4


def test_evict_scaled_value_block_is_chosen():
    c = rand_case(15, lens=(16, 16, 16), bs=4, d=16)
    vc = c["vc"].copy()
    for b in range(3):
        blk = c["bt"][b, 1 + b]
        vc[blk] = bf16_bits(bf16_vals(vc[blk]) * 0.125)
    s = oracle.score_tokens(c["kc"].ravel(), vc.ravel(), c["bs"] * c["Hkv"] * c["d"], c["bt"],
                            c["lens"], c["Hkv"], c["d"], c["bs"])
    ev, _, _ = oracle.select_evict_block(s, c["lens"], c["bs"])
    assert ev.tolist() == [1, 2, 3]


# ------------------------------------------------------------------ int8
def test_quantiser_golden_rows():
    with open(os.path.join(GOLDEN, "int8_rows.txt")) as f:
        rows = [ln for ln in f if ln.strip() and not ln.startswith("#")]
    for ln in rows:
        xs, s, qs = ln.split("|")
        x = np.array(xs.split(), np.float32)
        codes, scales = oracle.quantize_int8(bf16_bits(x)[None])
        assert scales[0] == np.float32(s)
        assert codes[0].tolist() == [int(v) for v in qs.split()]


def test_quantiser_range_and_error_bound():
    rng = np.random.default_rng(16)
    x = rng.standard_normal((500, 128)) * rng.uniform(0.01, 30, (500, 1))
    bits = bf16_bits(x)
    codes, scales = oracle.quantize_int8(bits)
    xv = bf16_vals(bits)
    assert np.abs(codes).max() <= 127
    assert (np.abs(codes).max(axis=1) == 127).all()          # the amax element maps to +-127
    deq = scales[:, None].astype(np.float64) * codes
    # |code - x/s| <= 1/2 plus the one fp32 rounding of x/s (|x/s| <= 127)
    bound = scales[:, None].astype(np.float64) * (0.5 + 127 * 2.0 ** -24)
    assert (np.abs(deq - xv) <= bound).all()


def test_int8_decode_equals_sdpa_on_dequantised_values():
    c = rand_case(17, Hq=8, Hkv=2, d=32, bs=4, N=20, lens=(4, 9, 14))
    kq, ks = oracle.quantize_int8(c["kc"])
    vq, vs = oracle.quantize_int8(c["vc"])
    out = oracle.paged_decode_int8(c["q"], kq.ravel(), vq.ravel(), ks.ravel(), vs.ravel(),
                                   c["bs"] * c["Hkv"] * c["d"], c["bt"], c["lens"], c["Hkv"],
                                   c["bs"], 1 / math.sqrt(c["d"]))
    kd = ks[..., None].astype(np.float64) * kq
    vd = vs[..., None].astype(np.float64) * vq
    B, Hq, Hkv, d = c["B"], c["Hq"], c["Hkv"], c["d"]
    q = bf16_vals(c["q"])
    for b in range(B):
        n = int(c["lens"][b])
        ids = c["bt"][b, : -(-n // c["bs"])]
        K = kd[ids].reshape(-1, Hkv, d)[:n]
        V = vd[ids].reshape(-1, Hkv, d)[:n]
        Kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
        Vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b]).unsqueeze(1), Kt, Vt, scale=1 / math.sqrt(d))[:, 0].numpy()
        np.testing.assert_allclose(out[b], o, rtol=1e-12, atol=1e-12)


def test_int8_append_matches_quantiser_and_slots():
    rng = np.random.default_rng(18)
    B, Hkv, d, bs, N, MB = 2, 2, 16, 4, 10, 3
    bt = np.array([[3, 7, -1], [1, 0, 9]], np.int32)
    kq = np.zeros(N * bs * Hkv * d, np.int8)
    vq = np.zeros_like(kq)
    ks = np.zeros(N * bs * Hkv, np.float32)
    vs = np.zeros_like(ks)
    kn = bf16_bits(rng.standard_normal((B, 3, Hkv, d)))
    vn = bf16_bits(rng.standard_normal((B, 3, Hkv, d)))
    pos = np.array([2, 7], np.int32)
    slots = oracle.append_kv_int8(kn, vn, kq, vq, ks, vs, bs * Hkv * d, bt, pos, bs)
    assert slots.tolist() == [[14, 15, 28], [3, 36, 37]]
    cq, cs = oracle.quantize_int8(kn)
    kq4 = kq.reshape(N * bs, Hkv, d)
    ks2 = ks.reshape(N * bs, Hkv)
    for b in range(B):
        for i in range(3):
            assert np.array_equal(kq4[slots[b, i]], cq[b, i])
            assert np.array_equal(ks2[slots[b, i]], cs[b, i])



def test_int8_score_equals_bf16_score_when_quantisation_is_exact():
    """Rows of integers in [-127, 127] whose amax is 127, times a power of two per row,
    quantise exactly (scale = that power of two, codes = the integers).  The score over
    the dequantised INT8 pools must then equal the bf16 score of the same values, and
    the numpy norm ratio; K and V rows carry different scales so that a scale taken from
    the wrong (token, head) row or from the other pool changes the result."""
    rng = np.random.default_rng(19)
    c = rand_case(19, lens=(5, 11, 16), d=16)
    N, bs, Hkv, d = c["N"], c["bs"], c["Hkv"], c["d"]

    def exact_rows():
        ints = rng.integers(-127, 128, (N, bs, Hkv, d)).astype(np.float64)
        ints[..., 0] = np.where(rng.random((N, bs, Hkv)) < 0.5, 127.0, -127.0)
        return ints * 2.0 ** rng.integers(-6, 3, (N, bs, Hkv, 1))

    kx, vx = exact_rows(), exact_rows()
    kb, vb = bf16_bits(kx), bf16_bits(vx)
    assert np.array_equal(bf16_vals(kb), kx) and np.array_equal(bf16_vals(vb), vx)
    kq, ks = oracle.quantize_int8(kb)
    vq, vs = oracle.quantize_int8(vb)
    assert np.array_equal(ks[..., None].astype(np.float64) * kq, kx)
    stride = bs * Hkv * d
    s8 = oracle.score_tokens_int8(kq.ravel(), vq.ravel(), ks.ravel(), vs.ravel(), stride, c["bt"],
                                  c["lens"], Hkv, d, bs)
    s16 = oracle.score_tokens(kb.ravel(), vb.ravel(), stride, c["bt"], c["lens"], Hkv, d, bs)
    for b in range(c["B"]):
        n = int(c["lens"][b])
        np.testing.assert_array_equal(s8[b, :n], s16[b, :n])
        assert np.isnan(s8[b, n:]).all()
        ids = c["bt"][b, : -(-n // bs)]
        K, V = kx[ids].reshape(-1, Hkv, d)[:n], vx[ids].reshape(-1, Hkv, d)[:n]
        ref = np.linalg.norm(V, axis=-1) / np.linalg.norm(K, axis=-1)
        np.testing.assert_allclose(s8[b, :n], ref, rtol=1e-13)


# ------------------------------------------------------------------ fp8 (e4m3)
def test_e4m3_golden_codes():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_values.txt")) as f:
        for ln in f:
            if ln.strip() and not ln.startswith("#"):
                v, c = ln.split()[:2]
                rows.append((float(v), int(c, 16)))
    x = np.array([v for v, _ in rows], np.float32)
    assert np.array_equal(bf16_vals(bf16_bits(x)), x.astype(np.float64))  # inputs exact in bf16
    codes = oracle.quantize_e4m3(bf16_bits(x))
    assert codes.tolist() == [c for _, c in rows]


def test_e4m3_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if (c & 0x7f) != 0x7f], np.uint8)
    vals = oracle.e4m3_values(codes)
    # every finite e4m3 value is exact in bf16 (3-bit mantissa, exponent in range)
    back = oracle.quantize_e4m3(bf16_bits(vals.astype(np.float32)))
    assert np.array_equal(back[codes != 0x80], codes[codes != 0x80])  # -0 encodes as 0x80
    pos = vals[(codes > 0) & (codes < 0x7f)]
    assert np.all(np.diff(pos) > 0) and pos.max() == 448.0 and pos.min() == 2.0 ** -9


def test_e4m3_matches_torch_cast_in_range():
    rng = np.random.default_rng(31)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (0.01, 1.0, 30.0, 150.0)])
    bits = bf16_bits(x)
    xv = bf16_vals(bits)
    keep = np.abs(xv) <= 448.0
    ours = oracle.quantize_e4m3(bits)[keep]
    ref = torch.as_tensor(xv[keep].astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8)
    assert np.array_equal(ours, ref.numpy())


def test_fp8_decode_equals_sdpa_on_decoded_values():
    c = rand_case(33, Hq=8, Hkv=2, d=32, bs=4, N=20, lens=(5, 9, 14))
    kq = oracle.quantize_e4m3(c["kc"])
    vq = oracle.quantize_e4m3(c["vc"])
    out = oracle.paged_decode_fp8(c["q"], kq.ravel(), vq.ravel(), c["bs"] * c["Hkv"] * c["d"],
                                  c["bt"], c["lens"], c["Hkv"], c["bs"], 1 / math.sqrt(c["d"]))
    kd, vd = oracle.e4m3_values(kq), oracle.e4m3_values(vq)
    B, Hq, Hkv, d = c["B"], c["Hq"], c["Hkv"], c["d"]
    q = bf16_vals(c["q"])
    for b in range(B):
        n = int(c["lens"][b])
        ids = c["bt"][b, : -(-n // c["bs"])]
        K = kd[ids].reshape(-1, Hkv, d)[:n]
        V = vd[ids].reshape(-1, Hkv, d)[:n]
        Kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
        Vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b]).unsqueeze(1), Kt, Vt, scale=1 / math.sqrt(d))[:, 0].numpy()
        np.testing.assert_allclose(out[b], o, rtol=1e-12, atol=1e-12)



def test_fp8_append_matches_torch_cast_and_slots():
    """The FP8 append stores torch's e4m3 cast of each new row at the slot the block
    table gives, and touches no other byte of either pool."""
    rng = np.random.default_rng(34)
    B, Hkv, d, bs, N = 2, 2, 16, 4, 10
    bt = np.array([[3, 7, -1], [1, 0, 9]], np.int32)
    kc = np.zeros(N * bs * Hkv * d, np.uint8)
    vc = np.zeros_like(kc)
    kn = bf16_bits(rng.standard_normal((B, 3, Hkv, d)) * 20)
    vn = bf16_bits(rng.standard_normal((B, 3, Hkv, d)) * 0.05)
    pos = np.array([2, 7], np.int32)
    slots = oracle.append_kv_fp8(kn, vn, kc, vc, bs * Hkv * d, bt, pos, bs)
    assert slots.tolist() == [[14, 15, 28], [3, 36, 37]]

    def cast(bits):
        return torch.as_tensor(bf16_vals(bits).astype(np.float32)).to(torch.float8_e4m3fn) \
            .view(torch.uint8).numpy()

    for pool, new in ((kc, kn), (vc, vn)):
        rows = pool.reshape(N * bs, Hkv, d)
        want = np.zeros_like(rows)
        for b in range(B):
            for i in range(3):
                want[slots[b, i]] = cast(new[b, i])
        assert np.array_equal(rows, want)


# ----------------------------------------------------------------------------- prefill stage
def test_prefill_score_closed_forms():
    """V = c_h K in head h gives a token score of mean_h |c_h|; K = 0 with V != 0
    gives +inf; K = V = 0 gives 0."""
    rng = np.random.default_rng(11)
    T, Hkv, d = 5, 4, 32
    k = rng.standard_normal((T, Hkv, d))
    c = np.array([0.5, -2.0, 0.25, 4.0])          # powers of two: c*K stays exact in bf16
    kb = bf16_bits(k)
    v = bf16_vals(kb).reshape(T, Hkv, d) * c[None, :, None]
    s = oracle.prefill_scores(kb.reshape(T, Hkv, d), bf16_bits(v).reshape(T, Hkv, d))
    assert np.allclose(s, np.abs(c).mean(), rtol=1e-15, atol=0)
    z = np.zeros((1, Hkv, d))
    one = np.ones((1, Hkv, d))
    assert oracle.prefill_scores(bf16_bits(z).reshape(1, Hkv, d),
                                 bf16_bits(one).reshape(1, Hkv, d))[0] == math.inf
    assert oracle.prefill_scores(bf16_bits(z).reshape(1, Hkv, d),
                                 bf16_bits(z).reshape(1, Hkv, d))[0] == 0.0


def test_prefill_score_is_head_mean_of_paged_score():
    """Written into a pool by the (pinned) append, the per-(token, head) paged
    scores averaged over heads equal the prefill scores."""
    rng = np.random.default_rng(12)
    T, Hkv, d, bs = 37, 2, 16, 8
    k = bf16_bits(rng.standard_normal((1, T, Hkv, d)))
    v = bf16_bits(rng.standard_normal((1, T, Hkv, d)) * 3)
    nb = -(-T // bs)
    bt = rng.permutation(nb).astype(np.int32)[None, :]
    stride = bs * Hkv * d
    kc = np.zeros(nb * stride, np.uint16)
    vc = np.zeros_like(kc)
    oracle.append_kv(k, v, kc, vc, stride, bt, np.zeros(1, np.int32), bs)
    paged = oracle.score_tokens(kc, vc, stride, bt, np.array([T], np.int32), Hkv, d, bs)
    s = oracle.prefill_scores(k[0], v[0])
    assert np.allclose(s, paged[0, :T].mean(axis=1), rtol=1e-14, atol=0)


def _keep_by_subsets(scores, budget):
    """Brute force: the unique kept set K of size budget such that every kept
    token outranks every evicted one, ranking by (value, index)."""
    import itertools
    n = len(scores)
    if n <= budget:
        return list(range(n))
    key = [((-math.inf if s != s else s), i) for i, s in enumerate(scores)]
    found = [c for c in itertools.combinations(range(n), budget)
             if min(key[i] for i in c) > max(key[i] for i in range(n) if i not in c)]
    assert len(found) == 1
    return list(found[0])


@pytest.mark.parametrize("seed", range(6))
def test_prefill_select_brute_force_over_subsets(seed):
    rng = np.random.default_rng(100 + seed)
    lens = [9, 3, 0, 7, 8]
    budget = 4
    # few distinct values: many ties
    vals = np.array([0.5, 1.0, 2.0, math.inf, math.nan, 0.0])
    scores = rng.choice(vals, size=sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    keep, kept = oracle.prefill_select(scores, cu, budget)
    for b, n in enumerate(lens):
        want = _keep_by_subsets(list(scores[cu[b]:cu[b + 1]]), budget)
        assert kept[b] == len(want)
        assert keep[b, :kept[b]].tolist() == want
        assert (keep[b, kept[b]:] == -1).all()


def test_prefill_select_closed_forms():
    cu = np.array([0, 10], np.int32)
    inc = np.arange(10, dtype=np.float64)
    assert oracle.prefill_select(inc, cu, 4)[0][0].tolist() == [6, 7, 8, 9]
    assert oracle.prefill_select(inc[::-1].copy(), cu, 4)[0][0].tolist() == [0, 1, 2, 3]
    # all equal: the latest tokens stay
    assert oracle.prefill_select(np.ones(10), cu, 3)[0][0].tolist() == [7, 8, 9]
    # planted low-importance tokens are the ones that go
    s = np.full(10, 2.0)
    s[[1, 4, 8]] = 0.1
    assert oracle.prefill_select(s, cu, 7)[0][0].tolist() == [0, 2, 3, 5, 6, 7, 9]
    # budget >= n keeps every token in order
    keep, kept = oracle.prefill_select(np.random.default_rng(0).random(10), cu, 16)
    assert kept[0] == 10 and keep[0, :10].tolist() == list(range(10))
    # -0 and +0 tie (index decides), NaN ranks below -inf... as -inf (index decides)
    s = np.array([0.0, -0.0, math.nan, -math.inf, 1.0])
    assert oracle.prefill_select(s, np.array([0, 5], np.int32), 3)[0][0].tolist() == [0, 1, 4]
    assert oracle.prefill_select(s, np.array([0, 5], np.int32), 4)[0][0].tolist() == [0, 1, 3, 4]


def test_prefill_pack_keep_all_equals_append():
    """With budget >= n the pack is the plain append of every prompt row."""
    rng = np.random.default_rng(13)
    lens = [5, 17, 16]
    Hkv, d, bs = 2, 8, 4
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    k = bf16_bits(rng.standard_normal((T, Hkv, d))).reshape(T, Hkv, d)
    v = bf16_bits(rng.standard_normal((T, Hkv, d))).reshape(T, Hkv, d)
    MB = max(-(-n // bs) for n in lens)
    N = 20
    perm = rng.permutation(N).astype(np.int32)
    bt = np.full((3, MB), -1, np.int32)
    c = 0
    for b, n in enumerate(lens):
        for j in range(-(-n // bs)):
            bt[b, j] = perm[c]
            c += 1
    stride = bs * Hkv * d
    kc1 = np.zeros(N * stride, np.uint16); vc1 = np.zeros_like(kc1)
    kc2 = np.zeros_like(kc1); vc2 = np.zeros_like(kc1)
    keep, kept = oracle.prefill_select(oracle.prefill_scores(k, v), cu, 64)
    oracle.prefill_pack(k, v, cu, keep, kept, kc1, vc1, stride, bt, bs)
    for b, n in enumerate(lens):
        oracle.append_kv(k[None, cu[b]:cu[b + 1]], v[None, cu[b]:cu[b + 1]], kc2, vc2, stride,
                         bt[b:b + 1], np.zeros(1, np.int32), bs)
    assert np.array_equal(kc1, kc2) and np.array_equal(vc1, vc2)


def test_prefill_pack_places_kept_rows_densely():
    """Logical gather of the packed pool returns exactly the kept rows in order."""
    rng = np.random.default_rng(14)
    lens = [23]
    Hkv, d, bs, budget = 1, 4, 4, 10
    cu = np.array([0, 23], np.int32)
    k = bf16_bits(rng.standard_normal((23, Hkv, d))).reshape(23, Hkv, d)
    v = bf16_bits(rng.standard_normal((23, Hkv, d))).reshape(23, Hkv, d)
    keep, kept = oracle.prefill_select(oracle.prefill_scores(k, v), cu, budget)
    bt = np.array([[5, 1, 3]], np.int32)
    stride = bs * Hkv * d
    kc = np.zeros(6 * stride, np.uint16); vc = np.zeros_like(kc)
    oracle.prefill_pack(k, v, cu, keep, kept, kc, vc, stride, bt, bs)
    for p in range(budget):
        blk, off = bt[0, p // bs], p % bs
        row = kc[blk * stride + off * Hkv * d: blk * stride + (off + 1) * Hkv * d]
        assert np.array_equal(row, k[keep[0, p]].ravel())
    # the two unused slots of the last block stay untouched
    assert not kc[3 * stride + 2 * d:3 * stride + 4 * d].any()


def test_evict_compact_preserves_token_to_slot_map():
    """Every token outside the evicted block keeps its physical slot, at a
    logical position bs lower when it came after the block; the freed id is the
    evicted block's; the table entries plus freed ids are a permutation of the old."""
    rng = np.random.default_rng(15)
    bs, MB = 4, 6
    lens = np.array([24, 17, 4, 3, 9], np.int32)
    evict = np.array([2, 0, 0, 0, 3], np.int32)      # seq 3 has no full block; 3 >= 9 // 4
    N = 40
    perm = rng.permutation(N).astype(np.int32)
    bt = np.full((5, MB), -1, np.int32)
    c = 0
    for b, n in enumerate(lens):
        for j in range(-(-int(n) // bs)):
            bt[b, j] = perm[c]
            c += 1
    nbt, nlen, freed = oracle.evict_compact(bt, lens, evict, bs)
    for b in range(5):
        j = int(evict[b])
        if not 0 <= j < lens[b] // bs:
            assert freed[b] == -1 and nlen[b] == lens[b] and (nbt[b] == bt[b]).all()
            continue
        assert freed[b] == bt[b, j] and nlen[b] == lens[b] - bs
        for p in range(lens[b]):
            if j * bs <= p < (j + 1) * bs:
                continue
            q = p - bs if p >= (j + 1) * bs else p
            assert oracle.slot(nbt[b], q, bs) == oracle.slot(bt[b], p, bs)
        old = sorted(x for x in bt[b] if x >= 0)
        new = sorted([x for x in nbt[b] if x >= 0] + [int(freed[b])])
        assert old == new
        assert (nbt[b, -(-int(nlen[b]) // bs):] == -1).all()


# ----------------------------------------------------------------------------- threshold policy
def _block_scores(consts, bs, Hkv, tail=0, tail_value=0.0):
    """One sequence whose full block j holds the constant score consts[j] in
    every (token, head) entry (so its mean is exactly consts[j]), plus a
    partial block of `tail` tokens."""
    MB = len(consts) + (1 if tail else 0)
    s = np.full((1, MB * bs, Hkv), np.nan)
    for j, c in enumerate(consts):
        s[0, j * bs:(j + 1) * bs] = c
    if tail:
        s[0, len(consts) * bs:len(consts) * bs + tail] = tail_value
    return s, np.array([len(consts) * bs + tail], np.int32)


def test_threshold_policy_trigger_boundary():
    s, lens = _block_scores([0.5, 0.01, 2.0], 4, 2)
    # usage 80 of 100 with eviction_ratio 0.2 is not above 80 %: nothing happens
    mask, count, _ = oracle.select_evict_threshold(s, lens, 4, 80, 100, 0.2, 0.1)
    assert count[0] == 0 and not mask.any()
    mask, count, _ = oracle.select_evict_threshold(s, lens, 4, 81, 100, 0.2, 0.1)
    assert count[0] == 1 and mask[0].tolist() == [0, 1, 0]


def test_threshold_policy_marks_every_block_below_threshold():
    # dyadic constants: every block sum and mean is exact in fp64
    consts = [0.5, 0.0625, 2.0, 0.09375, 0.125, 3.0, 0.1171875]
    s, lens = _block_scores(consts, 16, 8, tail=5, tail_value=0.001)
    mask, count, means = oracle.select_evict_threshold(s, lens, 16, 95, 100, 0.2, 0.125)
    # strictly below 0.125; the partial last block never counts however low it is
    assert mask[0].tolist() == [0, 1, 0, 1, 0, 0, 1, 0]
    assert count[0] == 3
    assert means[0, :7].tolist() == consts


def test_threshold_policy_without_low_blocks_is_the_decode_argmin():
    rng = np.random.default_rng(21)
    B, MB, bs, Hkv = 5, 9, 8, 2
    lens = np.array([72, 71, 8, 7, 40], np.int32)
    s = np.abs(rng.standard_normal((B, MB * bs, Hkv))) + 0.5
    mask, count, _ = oracle.select_evict_threshold(s, lens, bs, 99, 100, 0.2, 0.1)
    ev, _, _ = oracle.select_evict_block(s, lens, bs)
    for b in range(B):
        want = np.zeros(MB, np.uint8)
        if ev[b] >= 0:
            want[ev[b]] = 1
        assert mask[b].tolist() == want.tolist() and count[b] == int(ev[b] >= 0)


def test_compact_mask_single_block_equals_single_eviction():
    rng = np.random.default_rng(22)
    bs, MB = 4, 7
    lens = np.array([28, 27, 9, 3], np.int32)
    bt = np.full((4, MB), -1, np.int32)
    perm = rng.permutation(40).astype(np.int32)
    c = 0
    for b, n in enumerate(lens):
        m = -(-int(n) // bs)
        bt[b, :m] = perm[c:c + m]
        c += m
    evict = np.array([6, 3, 1, -1], np.int32)
    mask = np.zeros((4, MB), np.uint8)
    for b, j in enumerate(evict):
        if j >= 0:
            mask[b, j] = 1
    a_bt, a_len, a_fr = oracle.evict_compact(bt, lens, evict, bs)
    m_bt, m_len, m_fr = oracle.evict_compact_mask(bt, lens, mask, bs)
    assert np.array_equal(a_bt, m_bt) and np.array_equal(a_len, m_len)
    assert np.array_equal(m_fr[:, 0], a_fr) and (m_fr[:, 1:] == -1).all()


def test_compact_mask_preserves_token_to_slot_map():
    rng = np.random.default_rng(23)
    bs, MB = 4, 12
    lens = np.array([46, 48, 13], np.int32)
    bt = np.full((3, MB), -1, np.int32)
    perm = rng.permutation(60).astype(np.int32)
    c = 0
    for b, n in enumerate(lens):
        m = -(-int(n) // bs)
        bt[b, :m] = perm[c:c + m]
        c += m
    mask = np.zeros((3, MB), np.uint8)
    mask[0, [0, 3, 4, 10]] = 1
    mask[0, 11] = 1           # the partial block: ignored
    mask[1, [11, 5]] = 1      # includes the newest full block
    mask[2, 3] = 1            # partial: ignored
    nbt, nlen, fr = oracle.evict_compact_mask(bt, lens, mask, bs)
    for b in range(3):
        full = lens[b] // bs
        gone = [j for j in range(full) if mask[b, j]]
        assert nlen[b] == lens[b] - bs * len(gone)
        assert fr[b, :len(gone)].tolist() == [int(bt[b, j]) for j in gone]
        assert (fr[b, len(gone):] == -1).all()
        for p in range(lens[b]):
            j = p // bs
            if j in gone:
                continue
            q = p - bs * sum(1 for g in gone if g < j)
            assert oracle.slot(nbt[b], q, bs) == oracle.slot(bt[b], p, bs)
        assert (nbt[b, -(-int(nlen[b]) // bs):] == -1).all()


# ----------------------------------------------------------------------------- chunked prefill
def _prefill_case(seed, qlens, lens, Hq=8, Hkv=2, d=16, bs=4, N=60):
    c = rand_case(seed, B=len(lens), Hq=Hq, Hkv=Hkv, d=d, bs=bs, N=N, lens=tuple(lens))
    rng = np.random.default_rng(seed + 1000)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    c["qp"] = bf16_bits(rng.standard_normal((int(cu[-1]), Hq, d))).reshape(-1, Hq, d)
    c["cu"] = cu
    return c


def run_prefill(c):
    return oracle.paged_prefill(c["qp"], c["cu"], c["kc"].ravel(), c["vc"].ravel(),
                                c["bs"] * c["Hkv"] * c["d"], c["bt"], c["lens"], c["Hkv"],
                                c["bs"], 1.0 / math.sqrt(c["d"]))


@pytest.mark.parametrize("seed,Hq,Hkv,d,bs", [(1, 8, 2, 16, 4), (2, 4, 4, 8, 3), (3, 8, 1, 32, 5)])
def test_prefill_attention_equals_causal_sdpa(seed, Hq, Hkv, d, bs):
    """Against torch's fp64 scaled_dot_product_attention on the logically
    gathered K/V with the offset causal mask (query i of a q_len chunk at the
    end of n tokens sees tokens 0 .. n - q_len + i)."""
    qlens, lens = [5, 1, 13, 0], [23, 9, 13, 4]
    c = _prefill_case(seed, qlens, lens, Hq=Hq, Hkv=Hkv, d=d, bs=bs)
    got = run_prefill(c)
    for b, (ql, n) in enumerate(zip(qlens, lens)):
        if ql == 0:
            continue
        K, V = gather_logical(c, b)
        Kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
        Vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
        qt = torch.from_numpy(bf16_vals(c["qp"][c["cu"][b]:c["cu"][b + 1]])).permute(1, 0, 2)
        allowed = torch.arange(n)[None, :] <= (n - ql + torch.arange(ql))[:, None]
        o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=allowed,
                                                             scale=1 / math.sqrt(d))
        assert np.allclose(got[c["cu"][b]:c["cu"][b + 1]], o.permute(1, 0, 2).numpy(),
                           rtol=1e-12, atol=1e-13)


def test_prefill_attention_single_query_is_decode():
    lens = [23, 9, 13, 1]
    c = _prefill_case(5, [1, 1, 1, 1], lens)
    c["q"] = c["qp"].reshape(len(lens), c["Hq"], c["d"])
    assert np.array_equal(run_prefill(c), run_decode(c))


def test_prefill_attention_is_causal_and_invalid_rows_are_zero():
    c = _prefill_case(6, [6, 3], [20, 2])   # sequence 1 asks 3 queries of 2 tokens: invalid
    base = run_prefill(c)
    assert not base[6:].any()
    # change the last token of sequence 0: only its last query row moves
    b0_last = c["bt"][0, (20 - 1) // c["bs"]]
    c["kc"][b0_last, (20 - 1) % c["bs"]] = bf16_bits(np.full((c["Hkv"], c["d"]), 3.0))
    moved = run_prefill(c)
    assert np.array_equal(moved[:5], base[:5]) and not np.array_equal(moved[5], base[5])


# ----------------------------------------------------------------------------- mutation check
def test_mutation_check_still_applies_to_the_oracle():
    """Every planted mistake of tests/oracle_mutants.py still finds its text exactly
    once in oracle.c (so the mutation check keeps testing the current oracle), and one
    mutant, built and loaded through ORACLE_LIB, is rejected by a pin."""
    import importlib.util
    import subprocess
    import sys
    import tempfile
    here = os.path.dirname(os.path.abspath(__file__))
    spec = importlib.util.spec_from_file_location("oracle_mutants",
                                                  os.path.join(here, "oracle_mutants.py"))
    mut = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mut)
    src = open(mut.oracle_build.SRC).read()
    names = [m[0] for m in mut.MUTANTS]
    assert len(names) == len(set(names))
    for name, _, find, repl in mut.MUTANTS:
        assert src.count(find) == 1, name
        assert find != repl, name
    name, _, find, repl = next(m for m in mut.MUTANTS if m[0] == "gqa_mod")
    with tempfile.TemporaryDirectory() as tmp:
        c, so = os.path.join(tmp, "m.c"), os.path.join(tmp, "m.so")
        with open(c, "w") as f:
            f.write(src.replace(find, repl))
        mut.oracle_build.compile_c(c, so)
        r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                            os.path.join(here, "test_oracle_pins.py"), "-k",
                            "decode_equals_contiguous_sdpa"],
                           cwd=os.path.dirname(here), env=dict(os.environ, ORACLE_LIB=so),
                           capture_output=True, text=True)
        assert r.returncode != 0, r.stdout[-500:]
