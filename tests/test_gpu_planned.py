"""GPU: one partition plan serving several decode calls (pa_decode_prepare and the
planned decode calls) against the plain calls and the fp64 oracle.

The plan depends only on the context lengths and the sizes, which every layer of a
decode step shares; a planned call must give bit for bit what the plain call gives,
every time it is repeated on the kept plan, and a plan made for other sizes must be
refused on the device (flag, output untouched)."""
import numpy as np
import pytest
import torch

from helpers import Device, assert_attention_close, oracle_step
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu

C = W.CONFIGS
CASES = {
    # staged kernel, bf16, several layers over one plan
    "bf16": W.scaled(C["c3"], key="pl16", layers=3, batch=7, old_len_range=(1, 2500)),
    "bf16-d64": W.scaled(C["c2"], key="pl64", layers=3, batch=6,
                         old_lens=(1024, 1000, 17, 300, 1, 1039), score=False),
    "int8": W.scaled(C["c5"], key="pl8", layers=2, batch=5, old_lens=(300, 1, 16, 255, 512)),
    "fp8": W.scaled(C["c5"], key="plf8", layers=2, int8=False, fp8=True, batch=5,
                    old_lens=(300, 1, 16, 255, 512)),
    # full-batch shapes: c2's 32 sequences of 1024 tokens (5-6 pieces each) and 64 INT8
    # sequences of 512 (2-3 pieces each)
    "bf16-c2": W.scaled(C["c2"], key="plfu", layers=2, score=False),
    "int8-b64": W.scaled(C["c5"], key="plfu8", layers=2, batch=64, old_lens=(512,) * 64),
    # general-shape kernel (INT8 with d = 64): no device plan, the planned call is the plain one
    "int8-d64": W.scaled(C["c5"], key="pl8d64", layers=2, batch=3, head_dim=64,
                         old_lens=(70, 5, 200)),
}


def _planned_call(dev, layer, out):
    cfg = dev.wl.cfg
    if cfg.fp8:
        pk.pa_decode_fp8_planned(out, dev.q[layer], dev.k8[layer], dev.v8[layer], dev.bt,
                                 dev.ctx, dev.wl.scale, dev.err, dev.ws)
    elif cfg.int8:
        pk.pa_decode_int8_planned(out, dev.q[layer], dev.kq[layer], dev.vq[layer],
                                  dev.ks[layer], dev.vs[layer], dev.bt, dev.ctx, dev.wl.scale,
                                  dev.err, dev.ws)
    else:
        pk.pa_decode_planned(out, dev.q[layer], dev.k_pool[layer], dev.v_pool[layer], dev.bt,
                             dev.ctx, dev.wl.scale, dev.err, dev.ws)


def _pool0(dev):
    cfg = dev.wl.cfg
    return dev.k8[0] if cfg.fp8 else dev.kq[0] if cfg.int8 else dev.k_pool[0]


@pytest.mark.parametrize("key", list(CASES))
def test_planned_calls_equal_the_plain_calls_bitwise(key):
    wl = W.generate(CASES[key], "cpu")
    L = wl.q.shape[0]
    refs = [oracle_step(wl, l, range(wl.cfg.batch)) for l in range(L)]
    dev = Device(wl)
    if wl.cfg.int8 or wl.cfg.fp8:
        for l in range(L):
            dev.fill_int8_history(l)
    for l in range(L):            # plain calls: append + decode per layer
        dev.step(l)
    torch.cuda.synchronize()
    assert dev.err.item() == 0
    plain = dev.out.clone()
    for l in range(L):
        assert_attention_close(plain[l], refs[l]["out"], f"{key} layer {l}")
    # one plan for the step, then every layer (twice over) on the kept plan
    pk.pa_decode_prepare(dev.q[0], _pool0(dev), dev.bt, dev.ctx, dev.err, dev.ws)
    for rep in range(2):
        out = torch.full_like(dev.out, float("nan"))
        for l in range(L):
            _planned_call(dev, l, out[l])
        torch.cuda.synchronize()
        assert dev.err.item() == 0
        assert torch.equal(out, plain), (key, rep)


def test_a_plan_of_other_sizes_is_refused_on_the_device():
    wl = W.generate(CASES["bf16"], "cpu")
    dev = Device(wl)
    dev.step(0)
    torch.cuda.synchronize()
    # a plan for the first 4 sequences only, kept in the workspace
    pk.pa_decode_prepare(dev.q[0, :4], dev.k_pool[0], dev.bt[:4], dev.ctx[:4], dev.err, dev.ws)
    out = torch.full_like(dev.out[0], 7.0)
    pk.pa_decode_planned(out, dev.q[0], dev.k_pool[0], dev.v_pool[0], dev.bt, dev.ctx,
                         wl.scale, dev.err, dev.ws)
    torch.cuda.synchronize()
    assert dev.err.item() & pk.PA_DEV_BAD_PLAN
    assert (out == 7.0).all()
    # a zeroed workspace holds no plan either
    dev.err.zero_()
    dev.ws.zero_()
    pk.pa_decode_planned(out, dev.q[0], dev.k_pool[0], dev.v_pool[0], dev.bt, dev.ctx,
                         wl.scale, dev.err, dev.ws)
    torch.cuda.synchronize()
    assert dev.err.item() == pk.PA_DEV_BAD_PLAN
    assert (out == 7.0).all()
    # after a matching prepare the same call computes the plain result
    dev.err.zero_()
    pk.pa_decode_prepare(dev.q[0], dev.k_pool[0], dev.bt, dev.ctx, dev.err, dev.ws)
    pk.pa_decode_planned(out, dev.q[0], dev.k_pool[0], dev.v_pool[0], dev.bt, dev.ctx,
                         wl.scale, dev.err, dev.ws)
    torch.cuda.synchronize()
    assert dev.err.item() == 0
    assert torch.equal(out, dev.out[0])
    assert np.isfinite(out.float().cpu().numpy()).all()
