"""GPU: the merge of the staged decode's partial results, against the fp64 oracle.

With the automatic split a sequence's pieces write (acc, m, l) partials that a
merge kernel combines: one warp per output row when the rows have few partials on
average (at most 8 per sequence), one CTA per row otherwise.  The cases cover a
row with more than 32 partials in the warp-per-row merge (it takes them 32 at a
time), two consumer warps per kv head (two partials per piece), empty sequences
(a zero row), the INT8 and FP8 consumers, and repeated calls (the merge is in
slot order: bit-identical results)."""
import numpy as np
import pytest
import torch

from helpers import Device, assert_attention_close, oracle_step
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu

C = W.CONFIGS

CASES = {
    # Llama-3.2-1B shape at its batch (32 x 1024 tokens): 5-6 pieces per sequence, G = 4
    "c2": W.scaled(C["c2"], key="fm2", layers=1, score=False),
    # Hkv = 4: two consumer warps per kv head (partials = 2 per piece), G = 8, d = 128;
    # empty sequences among them (no append)
    "wph2": W.scaled(C["c3"], key="fmw2", layers=1, batch=160, hq=32, hkv=4,
                     old_lens=tuple(0 if i % 37 == 5 else 40 + (i * 53) % 700 for i in range(160)),
                     append=False, outlier_frac=0.0),
    # one long sequence among short ones, G = 1: that sequence's rows are merged from
    # about 145 partials by the warp-per-row merge
    "long-row": W.scaled(C["c3"], key="fmlr", layers=1, batch=64, hq=8, hkv=8,
                         old_lens=(60000,) + (16,) * 62 + (0,), append=False,
                         outlier_frac=0.0),
    # G = 8 with about ten pieces per long sequence and one or two per short one
    "groups": W.scaled(C["c3"], key="fmgr", layers=1, batch=64, hq=64, hkv=8,
                       old_lens=tuple(8192 if i % 4 == 0 else 64 for i in range(64)),
                       outlier_frac=0.0),
    # the INT8 and FP8 consumers (d = 128, G = 8)
    "int8": W.scaled(C["c5"], key="fmi8", batch=64, old_lens=(512,) * 64),
    "fp8": W.scaled(C["c5"], key="fmf8", int8=False, fp8=True, batch=64,
                    old_lens=tuple(300 + (i * 97) % 900 for i in range(64))),
}


@pytest.mark.parametrize("key", list(CASES))
def test_merged_partials_match_the_oracle(key):
    wl = W.generate(CASES[key], "cpu")
    cfg = wl.cfg
    ref = oracle_step(wl, 0, range(cfg.batch))
    dev = Device(wl)
    if cfg.int8 or cfg.fp8:
        dev.fill_int8_history(0)
    outs = []
    # a repeated step appends the same token to the same slot again
    for rep in range(3):
        dev.out.fill_(float("nan"))
        dev.step(0)
        torch.cuda.synchronize()
        assert dev.err.item() == 0, f"device error flag {dev.err.item()}"
        assert_attention_close(dev.out[0], ref["out"], f"{key} call {rep}")
        outs.append(dev.out[0].clone())
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    lens = np.asarray(wl.ctx_lens)
    for b in np.nonzero(lens == 0)[0]:
        assert (dev.out[0, b] == 0).all(), f"empty sequence {b} must give a zero row"


def test_split_decode_is_three_launches():
    """Plan, decode and merge kernels per call whenever a sequence is split."""
    cfg = C["c4"]
    assert pk.pa_decode_plan(cfg.batch, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block_size,
                             131072 // 256)[2] == 3
