"""The seeded synthetic inputs match the recipe the design states: shapes and lengths
of each workload, seeds 396 + index, the c3 outlier channels, pool sizing and the
shuffled free list, and the chunked-prefill layout (small stand-ins of the same
generators where the full size would not fit a CPU test)."""
import dataclasses

import numpy as np

from paged_kv_cache_396_b200 import workloads as W


def test_config_shapes_and_seeds():
    C = W.CONFIGS
    assert [C[k].seed for k in ("c1", "c2", "c3", "c4", "c5")] == [396, 397, 398, 399, 400]
    assert (C["c2"].layers, C["c2"].batch, C["c2"].hq, C["c2"].hkv, C["c2"].head_dim) == (16, 32, 32, 8, 64)
    assert C["c2"].old_lens == (1024,) * 32 and C["c2"].score
    assert (C["c3"].layers, C["c3"].batch, C["c3"].hq, C["c3"].hkv, C["c3"].head_dim) == (32, 64, 32, 8, 128)
    assert C["c3"].old_len_range == (512, 8192) and C["c3"].outlier_frac == 0.01
    assert C["c4"].block_size == 256 and C["c4"].old_lens == (131072,) * 4 and not C["c4"].append
    assert C["c5"].int8 and C["c5"].hq == 64 and C["c5"].old_lens == (4096,) * 128
    p1, p2 = W.PREFILL["p1"], W.CHUNKED["p2"]
    assert (p1.seed, p2.seed) == (401, 402)
    assert p1.batch == 32 and set(p1.prompt_lens) == {8192} and p1.budget == 1024
    assert (p1.hkv, p1.head_dim, p1.block_size) == (8, 128, 16)
    assert (p2.batch, p2.ctx_len, p2.chunk, p2.hq, p2.hkv, p2.head_dim) == (4, 8192, 512, 32, 8, 128)


def test_tables_use_a_shuffled_free_list_and_spare_pool():
    cfg = dataclasses.replace(W.CONFIGS["c3"], layers=1, batch=6, old_len_range=(1, 700))
    wl = W.generate(cfg, "cpu")
    lens = wl.ctx_lens.astype(np.int64)
    assert np.array_equal(lens, wl.old_lens + 1) and np.array_equal(wl.positions, wl.old_lens)
    need = [-(-int(n) // cfg.block_size) for n in lens]
    used = np.concatenate([wl.block_tables[b, :need[b]] for b in range(cfg.batch)])
    assert len(set(used.tolist())) == len(used)                     # no block shared
    assert used.min() >= 0 and used.max() < wl.num_blocks
    assert (wl.block_tables[wl.block_tables >= 0].size == used.size)
    assert wl.num_blocks >= int(np.ceil(1.1 * used.size)) - 1      # ~10 % spare
    assert not np.array_equal(np.sort(used), used)                  # shuffled, not in order


def test_c3_outlier_channels_are_one_percent_scaled_by_eight():
    cfg = dataclasses.replace(W.CONFIGS["c3"], layers=1, batch=2, old_len_range=(200, 300))
    wl = W.generate(cfg, "cpu")
    pairs = wl.outliers[0]
    assert len(pairs) == round(0.01 * cfg.hkv * cfg.head_dim)       # 10 of 1024, rounded
    k = wl.k_pool[0].float()
    used = wl.block_tables[0, 0]
    blk = k[used].reshape(-1, cfg.hkv, cfg.head_dim)
    rms = blk.pow(2).mean(0).sqrt()
    for h, c in pairs:
        assert rms[h, c] > 4.0                                      # N(0,1) x 8
    mask = np.ones((cfg.hkv, cfg.head_dim), bool)
    for h, c in pairs:
        mask[h, c] = False
    assert float(rms[mask].mean()) < 1.5


def test_same_seed_same_inputs():
    cfg = dataclasses.replace(W.CONFIGS["c2"], layers=1, batch=3, old_lens=(40, 1, 77))
    a, b = W.generate(cfg, "cpu"), W.generate(cfg, "cpu")
    assert np.array_equal(a.block_tables, b.block_tables)
    assert np.array_equal(W.bits(a.q), W.bits(b.q))
