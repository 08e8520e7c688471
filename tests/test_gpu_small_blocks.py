"""Block sizes below 12 tokens.

The C ABI takes any block size from 1 token up.  Sizes that are not multiples of 16
go to the general decode kernel, the general chunked-prefill kernel and the
per-token append, score and selection kernels.  Each case runs the append, the
decode and (bf16) the norm-ratio scores and the lowest-mean block over block sizes
1, 2, 3, 5 and 8.  Slots are compared bit for bit and outputs element by element
with the fp64 oracle ([VKV] §2.1 append_slot, §2.2 paged_attention_forward; [KVL]
"PagedEviction 块级驱逐机制").  The chunked prefill over the same sizes is compared
with the oracle too ([KVP] "Chunked prefill：让 prefill 不阻塞 decode")."""
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
SIZES = (1, 2, 3, 5, 8)


def _cfg(bs, kv, d, seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(2, 12))
    special = [0, 1, bs - 1, bs, bs + 1, 2 * bs, 127, 128]
    lens = tuple(max(0, int(rng.choice(special))) if rng.random() < 0.4
                 else int(rng.integers(1, 300)) for _ in range(B))
    base = C["c5"] if kv == "int8" else C["c3"]
    return W.scaled(base, key=f"sb{bs}{kv}{d}", layers=1, batch=B, hq=16, hkv=4, head_dim=d,
                    block_size=bs, old_lens=lens, old_len_range=(), append=True,
                    outlier_frac=0.0, int8=kv == "int8", fp8=kv == "fp8", nano_layout=False,
                    score=False, pool_blocks=None, seed=seed)


@pytest.mark.parametrize("bs", SIZES)
@pytest.mark.parametrize("kv,d", [("bf16", 64), ("bf16", 128), ("int8", 128), ("fp8", 128)])
def test_small_block_append_decode(bs, kv, d):
    cfg = _cfg(bs, kv, d, 8000 + 10 * bs + d + {"bf16": 0, "int8": 1, "fp8": 2}[kv])
    wl = W.generate(cfg, "cpu")
    score = kv == "bf16"
    ref = oracle_step(wl, 0, range(cfg.batch), score=score)
    dev = Device(wl)
    if cfg.int8 or cfg.fp8:
        dev.fill_int8_history(0)
    res = dev.step(0, score=score)
    torch.cuda.synchronize()
    assert dev.err.item() == 0, f"device error flag {dev.err.item()}"
    # the oracle's slots are ids in its compact copy of the pool: map them back
    bt_c, expect = ref["compact"]["block_tables"], np.empty_like(ref["slots"])
    for b in range(cfg.batch):
        blk, off = divmod(int(ref["slots"][b, 0]), bs)
        j = int(np.nonzero(bt_c[b] == blk)[0][0])
        expect[b, 0] = int(wl.block_tables[b, j]) * bs + off
    assert np.array_equal(dev.slots.cpu().numpy(), expect), "slots"
    assert_attention_close(dev.out[0], ref["out"], f"bs {bs} {kv} d {d}: {cfg.old_lens}")
    if score:
        got = res["scores"].cpu().numpy()
        for b in range(cfg.batch):
            n = int(wl.ctx_lens[b])
            assert_scores_close(got[b, :n], ref["scores"][b, :n], f"bs {bs} seq {b}")
        assert_evict_consistent(res["evict"].cpu().numpy(), ref["evict"], ref["means"],
                                ref["gap"], f"bs {bs}")


@pytest.mark.parametrize("bs", SIZES)
@pytest.mark.parametrize("balanced", [False, True])
def test_small_block_chunked_prefill(bs, balanced):
    rng = np.random.default_rng(8100 + bs)
    g = torch.Generator().manual_seed(8100 + bs)
    Hq, Hkv, d = 16, 4, 128
    lens = [int(rng.integers(1, 400)) for _ in range(3)] + [bs, 1]
    qlens = [int(rng.integers(0, n + 1)) for n in lens]
    nb = [-(-n // bs) for n in lens]
    N = sum(nb) + 3
    perm = rng.permutation(N).astype(np.int32)
    bt = np.full((len(lens), max(nb)), -1, np.int32)
    c = 0
    for b, m in enumerate(nb):
        bt[b, :m] = perm[c:c + m]
        c += m
    k = torch.randn(N, bs, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(N, bs, Hkv, d, generator=g).to(torch.bfloat16)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = torch.randn(int(cu[-1]), Hq, d, generator=g).to(torch.bfloat16)
    dev = "cuda"
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    mq = max(qlens)
    ws = pk.alloc_prefill_workspace(len(lens), Hq, Hkv, d, bs, mq, dev) if balanced else None
    pk.pa_prefill_attention(out, q.to(dev), torch.as_tensor(cu, device=dev), mq, k.to(dev),
                            v.to(dev), torch.as_tensor(bt, device=dev),
                            torch.as_tensor(np.asarray(lens, np.int32), device=dev), d ** -0.5,
                            err, workspace=ws)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oracle.paged_prefill(W.bits(q), cu, W.bits(k).ravel(), W.bits(v).ravel(),
                               bs * Hkv * d, bt, np.asarray(lens, np.int32), Hkv, bs, d ** -0.5)
    assert_attention_close(out, ref, f"bs {bs}: lens {lens} qlens {qlens}")
