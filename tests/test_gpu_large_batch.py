"""Batches larger than the plan kernels' shared-memory caches.

The balanced decode plan keeps the lengths and starts of the first 1024 sequences
in shared memory and reads the rest from global memory.  The chunked-prefill plan
keeps the tile counts of the first 4096 items.  Serving batches past those sizes
take the other path.  These cases run decode over 1100 to 2100 sequences (bf16
d = 128 with the automatic and an explicit split, bf16 d = 64, INT8, e4m3), and
chunked prefill over 4800 items in both modes.  Lengths mix zero, one token, tile
and block multiples and ragged tails.  Every output element is compared with the
fp64 oracle at the stated tolerance ([KVP] "PagedAttention 的算子"; [VKV] §2.2 and
§6.1; [KVP] "Chunked prefill：让 prefill 不阻塞 decode")."""
import numpy as np
import pytest
import torch

import oracle
from helpers import Device, assert_attention_close, oracle_step
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu

C = W.CONFIGS


def _lens(rng, B, hi):
    special = [0, 1, 15, 16, 17, 127, 128, 129, 255, 256, 257]
    return tuple(int(rng.choice(special)) if rng.random() < 0.3 else int(rng.integers(1, hi))
                 for _ in range(B))


CASES = {
    # name: (base config, batch, q heads, kv heads, head dim, kv storage, split, lengths
    # below); the INT8 and e4m3 cases keep a bf16 history of the longest length per
    # sequence on the host, so their lengths stay shorter
    "bf16-d128-b1500": ("c3", 1500, 32, 8, 128, "bf16", 0, 400),
    "bf16-d128-b1500-split2": ("c3", 1500, 32, 8, 128, "bf16", 2, 400),
    "bf16-d64-b2100": ("c2", 2100, 32, 8, 64, "bf16", 0, 400),
    "int8-b1100": ("c5", 1100, 64, 8, 128, "int8", 0, 200),
    "fp8-b1100": ("c5", 1100, 32, 8, 128, "fp8", 0, 200),
}


@pytest.mark.parametrize("name", list(CASES))
def test_decode_over_more_sequences_than_the_plan_caches(name):
    base, B, hq, hkv, d, kv, splits, hi = CASES[name]
    seed = 7100 + sum(map(ord, name))
    lens = _lens(np.random.default_rng(seed), B, hi)
    cfg = W.scaled(C[base], key=f"lb-{name}", layers=1, batch=B, hq=hq, hkv=hkv, head_dim=d,
                   block_size=16, old_lens=lens, old_len_range=(), append=True,
                   outlier_frac=0.0, int8=kv == "int8", fp8=kv == "fp8", nano_layout=False,
                   score=False, pool_blocks=None, seed=seed)
    wl = W.generate(cfg, "cpu")
    ref = oracle_step(wl, 0, range(B))
    dev = Device(wl, num_splits=splits)
    if cfg.int8 or cfg.fp8:
        dev.fill_int8_history(0)
    dev.step(0)
    torch.cuda.synchronize()
    assert dev.err.item() == 0, f"device error flag {dev.err.item()}"
    assert_attention_close(dev.out[0], ref["out"], f"{name}: {B} sequences")


@pytest.mark.parametrize("balanced", [False, True])
def test_chunked_prefill_over_more_items_than_the_plan_cache(balanced):
    """600 sequences x 8 kv heads = 4800 items (one 256-row item per chunk of at most
    64 tokens at G = 4), past the plan's 4096 cached tile counts."""
    rng = np.random.default_rng(7300)
    g = torch.Generator().manual_seed(7300)
    B, Hq, Hkv, d, bs = 600, 32, 8, 128, 16
    lens = [max(1, x) for x in _lens(rng, B, 300)]
    qlens = [int(rng.integers(0, min(n, 16) + 1)) for n in lens]
    nb = [-(-n // bs) for n in lens]
    N = sum(nb) + 4
    perm = rng.permutation(N).astype(np.int32)
    bt = np.full((B, max(nb)), -1, np.int32)
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
    ws = pk.alloc_prefill_workspace(B, Hq, Hkv, d, bs, max(qlens), dev) if balanced else None
    pk.pa_prefill_attention(out, q.to(dev), torch.as_tensor(cu, device=dev), max(qlens),
                            k.to(dev), v.to(dev), torch.as_tensor(bt, device=dev),
                            torch.as_tensor(np.asarray(lens, np.int32), device=dev), d ** -0.5,
                            err, workspace=ws)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oracle.paged_prefill(W.bits(q), cu, W.bits(k).ravel(), W.bits(v).ravel(),
                               bs * Hkv * d, bt, np.asarray(lens, np.int32), Hkv, bs, d ** -0.5)
    assert_attention_close(out, ref, f"chunked prefill over {B * Hkv} items")
