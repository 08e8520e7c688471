"""GPU: seeded random decode shapes against the fp64 oracle.

Each case draws a batch size, the GQA shape, the head size, the block size, the
KV storage (bf16, INT8, e4m3), a split count and per-sequence lengths (zero,
one token, exact tile and block multiples, ragged tails) from a fixed seed,
runs the append and the decode through the C ABI, and compares every output
element with the oracle at the stated tolerance.  The cases reach both decode
kernels (the staged one for block sizes that are multiples of 16 and
Hkv in {1, 2, 4, 8}, the general one otherwise), the automatic split with both
merge kernels, and explicit splits."""
import numpy as np
import pytest
import torch

from helpers import Device, assert_attention_close, oracle_step
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu

C = W.CONFIGS


def _case(i):
    rng = np.random.default_rng(9000 + i)
    kv = ("bf16", "int8", "fp8")[i % 3]
    hkv = int(rng.choice([1, 2, 4, 8]))
    g = int(rng.choice([1, 2, 4, 8, 16]))
    d = 128 if kv != "bf16" and i % 2 == 0 else int(rng.choice([64, 128]))
    bs = int(rng.choice([16, 16, 32, 12, 256]))
    B = int(rng.integers(1, 40))
    special = [0, 1, 15, 16, 17, bs - 1, bs, bs + 1, 255, 256, 257]
    lens = [int(rng.choice(special)) if rng.random() < 0.4 else int(rng.integers(1, 3000))
            for _ in range(B)]
    splits = int(rng.choice([0, 0, 0, 1, 3]))
    base = C["c5"] if kv == "int8" else C["c3"]
    cfg = W.scaled(base, key=f"rnd{i}", layers=1, batch=B, hq=hkv * g, hkv=hkv, head_dim=d,
                   block_size=bs, old_lens=tuple(lens), old_len_range=(), append=True,
                   outlier_frac=0.0, int8=kv == "int8", fp8=kv == "fp8", nano_layout=False,
                   pool_blocks=None, seed=9000 + i)
    return cfg, splits


@pytest.mark.parametrize("i", range(64))
def test_random_shape_matches_the_oracle(i):
    cfg, splits = _case(i)
    wl = W.generate(cfg, "cpu")
    ref = oracle_step(wl, 0, range(cfg.batch))
    dev = Device(wl, num_splits=splits)
    if cfg.int8 or cfg.fp8:
        dev.fill_int8_history(0)
    dev.step(0)
    torch.cuda.synchronize()
    assert dev.err.item() == 0, f"device error flag {dev.err.item()}"
    assert_attention_close(dev.out[0], ref["out"], f"case {i}: {cfg}")
