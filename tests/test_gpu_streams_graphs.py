"""The calls as a serving runtime issues them: on streams of its own and inside CUDA
graphs.

- Two decode steps of different batches on two streams at once, each with its own
  workspace and error flag, give the same bits as the same steps one after the other
  on the default stream.
- The chunked-prefill call (grid mode: one launch; balanced mode: the plan and two
  attention launches chained by programmatic dependent launch) and the planned INT8
  decode (plan once, then the decode call) are captured in CUDA graphs.  Replays give
  the same bits as eager calls, also after the inputs change in place between
  replays.
The eager results themselves are checked against the oracle by the parity tests."""
import numpy as np
import pytest
import torch

from helpers import Device, assert_attention_close, oracle_step
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu

C = W.CONFIGS


def _bits(t):
    return t.view(torch.int16).clone()


def _decode_case(key, B, seed):
    cfg = W.scaled(C["c3"], key=key, layers=1, batch=B, old_len_range=(1, 3000),
                   outlier_frac=0.0, seed=seed)
    return W.generate(cfg, "cpu")


def test_decode_steps_on_two_streams_at_once():
    wls = [_decode_case("st1", 9, 61), _decode_case("st2", 23, 62)]
    # one after the other, default stream
    seq = []
    for wl in wls:
        dev = Device(wl)
        dev.step(0)
        torch.cuda.synchronize()
        assert dev.err.item() == 0
        seq.append(_bits(dev.out[0]))
    # both at once, a stream each (fresh device copies: the append writes the pools)
    devs = [Device(wl) for wl in wls]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    torch.cuda.synchronize()
    for rep in range(3):
        for dev, s in zip(devs, streams):
            with torch.cuda.stream(s):
                dev.step(0)
        torch.cuda.synchronize()
        for i, dev in enumerate(devs):
            assert dev.err.item() == 0
            assert torch.equal(_bits(dev.out[0]), seq[i]), (rep, i)
    ref = oracle_step(wls[1], 0, range(wls[1].cfg.batch))
    assert_attention_close(devs[1].out[0], ref["out"], "decode on a side stream")


@pytest.mark.parametrize("balanced", [False, True])
def test_chunked_prefill_replays_in_a_cuda_graph(balanced):
    g = torch.Generator().manual_seed(63)
    rng = np.random.default_rng(63)
    Hq, Hkv, d, bs = 32, 8, 128, 16
    lens, qlens = [2048, 700, 37, 5, 1100], [512, 1, 37, 0, 100]
    nb = [-(-n // bs) for n in lens]
    N = sum(nb) + 4
    perm = rng.permutation(N).astype(np.int32)
    bt = np.full((len(lens), max(nb)), -1, np.int32)
    c = 0
    for b, m in enumerate(nb):
        bt[b, :m] = perm[c:c + m]
        c += m
    dev = "cuda"
    k = torch.randn(N, bs, Hkv, d, generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn(N, bs, Hkv, d, generator=g).to(torch.bfloat16).to(dev)
    cu = torch.as_tensor(np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32), device=dev)
    T = int(cu[-1])
    qs = [torch.randn(T, Hq, d, generator=g).to(torch.bfloat16).to(dev) for _ in range(2)]
    btd = torch.as_tensor(bt, device=dev)
    ctx = torch.as_tensor(np.asarray(lens, np.int32), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = pk.alloc_prefill_workspace(len(lens), Hq, Hkv, d, bs, max(qlens), dev) \
        if balanced else None
    q = qs[0].clone()
    out = torch.empty_like(q)

    def call():
        pk.pa_prefill_attention(out, q, cu, max(qlens), k, v, btd, ctx, d ** -0.5, err,
                                workspace=ws)

    eager = []
    for qi in qs:
        q.copy_(qi)
        call()
        torch.cuda.synchronize()
        eager.append(_bits(out))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for _ in range(2):
        for qi, ref in zip(qs, eager):
            q.copy_(qi)
            out.fill_(float("nan"))
            graph.replay()
            torch.cuda.synchronize()
            assert torch.equal(_bits(out), ref)
    assert err.item() == 0


def test_planned_int8_decode_replays_in_a_cuda_graph():
    cfg = W.scaled(C["c5"], key="gi8", batch=12, old_lens=(4096, 1, 17, 300, 2000, 513, 64,
                                                              1000, 3000, 128, 129, 777))
    wl = W.generate(cfg, "cpu")
    dev = Device(wl)
    dev.fill_int8_history(0)
    torch.cuda.synchronize()
    args = (dev.kq[0], dev.vq[0], dev.ks[0], dev.vs[0], dev.bt, dev.ctx, wl.scale, dev.err,
            dev.ws)
    q = dev.q[0].clone()
    out = torch.empty_like(q)

    def call():
        pk.pa_decode_prepare(q, dev.kq[0], dev.bt, dev.ctx, dev.err, dev.ws)
        pk.pa_decode_int8_planned(out, q, *args)

    q2 = torch.randn(q.shape, generator=torch.Generator().manual_seed(64)).to(q)
    eager = []
    for qi in (dev.q[0], q2):
        q.copy_(qi)
        call()
        torch.cuda.synchronize()
        eager.append(_bits(out))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for qi, ref in zip((dev.q[0], q2), eager):
        q.copy_(qi)
        out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(_bits(out), ref)
    assert dev.err.item() == 0
