"""Contexts far past the benchmark's 128K.

Decode over sequences of 1 048 576 and 300 000 tokens in the nano-vLLM layout
(block 256; [NANO] "物理内存布局：连续张量与分块策略").  The automatic split then
cuts each sequence into many partitions and the merge takes its warp-split path.
Every output element is compared with the fp64 oracle ([KVP] "PagedAttention 的算子").

Chunked prefill of the last 512 tokens of a 262 144-token context (block 16,
Llama-3-8B shape), in both modes.  An item there spans 2048 K/V tiles, and the
balanced mode cuts it across several CTAs whose partial results the last part
merges.  Causality makes chunk row i a decode over its own p + 1 tokens, so sampled
rows are compared with the decode oracle at their positions ([KVP] "Chunked
prefill：让 prefill 不阻塞 decode")."""
import numpy as np
import pytest
import torch

import oracle
from helpers import Device, assert_attention_close, oracle_step
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _free():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def test_decode_over_a_million_tokens():
    cfg = W.scaled(W.CONFIGS["c4"], key="lc1m", batch=2, old_lens=(1048576, 300000), seed=41)
    wl = W.generate(cfg, torch.device("cuda"))
    ref = oracle_step(wl, 0, range(cfg.batch))
    dev = Device(wl)
    dev.step(0)
    torch.cuda.synchronize()
    assert dev.err.item() == 0
    ns = pk.workspace_plan(dev.ws, cfg.batch)[2]
    assert max(ns) > 32          # more partials per row than the merge's per-thread path
    assert_attention_close(dev.out[0], ref["out"], "decode over 1M + 300K tokens")


@pytest.mark.parametrize("balanced", [False, True])
def test_chunked_prefill_at_the_end_of_a_256k_context(balanced):
    Hq, Hkv, d, bs = 32, 8, 128, 16
    n, ql = 262144, 512
    dev = "cuda"
    g = torch.Generator(device=dev).manual_seed(43)
    rng = np.random.default_rng(43)
    nb = n // bs
    N = nb + 8
    bt = rng.permutation(N)[:nb].astype(np.int32)[None, :]
    k = torch.randn(N, bs, Hkv, d, generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn(N, bs, Hkv, d, generator=g, device=dev).to(torch.bfloat16)
    q = torch.randn(ql, Hq, d, generator=g, device=dev).to(torch.bfloat16)
    cu = torch.as_tensor([0, ql], dtype=torch.int32, device=dev)
    out = torch.full_like(q, float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = pk.alloc_prefill_workspace(1, Hq, Hkv, d, bs, ql, dev) if balanced else None
    pk.pa_prefill_attention(out, q, cu, ql, k, v, torch.as_tensor(bt, device=dev),
                            torch.as_tensor([n], dtype=torch.int32, device=dev), d ** -0.5,
                            err, workspace=ws)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert torch.isfinite(out.float()).all()
    kb, vb = W.bits(k).ravel(), W.bits(v).ravel()
    out = out.cpu()
    for i in (0, 137, 255, 256, 511):
        p = n - ql + i
        ref = oracle.paged_decode(W.bits(q[i:i + 1]), kb, vb, bs * Hkv * d, bt,
                                  np.array([p + 1], np.int32), Hkv, bs, d ** -0.5)
        assert_attention_close(out[i:i + 1], ref, f"chunk row {i} at position {p}")
