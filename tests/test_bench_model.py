"""The roofline numerators bench.py reports, pinned by counting: the chunked-prefill
FLOPs against the closed form of the causal count, and the decode's algorithmic
bytes against the marginal cost of one more cached token."""
import dataclasses

import numpy as np
import pytest

import bench
from paged_kv_cache_396_b200 import workloads as W


def test_chunk_flops_is_the_causal_count():
    cfg = W.CHUNKED["p2"]
    # query i of the chunk sees ctx - chunk + i + 1 tokens; QK^T and PV are 2 d flops
    # each per (row, token, head)
    n, c = cfg.ctx_len, cfg.chunk
    seen = c * (n - c + 1) + c * (c - 1) // 2
    assert bench.chunk_flops(cfg) == 4 * cfg.head_dim * cfg.hq * cfg.batch * seen
    # brute force on a small chunk
    small = dataclasses.replace(cfg, ctx_len=40, chunk=7, batch=2)
    brute = sum(4 * small.head_dim * small.hq * (40 - 7 + i + 1) for i in range(7)) * 2
    assert bench.chunk_flops(small) == brute


def test_decode_bytes_count_each_cached_token_once():
    for key, elt, scales in (("c3", 2, 0), ("c5", 1, 8)):
        cfg = W.CONFIGS[key]
        lens = np.array([100, 17, 16], np.int64)
        base = bench.decode_algorithmic_bytes(dataclasses.replace(cfg, batch=3), lens, 0)
        for b in range(3):
            more = lens.copy()
            more[b] += 1
            grown = bench.decode_algorithmic_bytes(dataclasses.replace(cfg, batch=3), more, 0)
            new_block = 4 if lens[b] % cfg.block_size == 0 else 0
            per_token = cfg.hkv * cfg.head_dim * 2 * elt + cfg.hkv * scales
            assert grown - base == per_token + new_block, (key, b)


def test_decode_bytes_include_partials_both_ways():
    cfg = dataclasses.replace(W.CONFIGS["c3"], batch=2)
    lens = np.array([500, 300], np.int64)
    a = bench.decode_algorithmic_bytes(cfg, lens, 0)
    b = bench.decode_algorithmic_bytes(cfg, lens, 3)
    # three partition slots of Hq rows: (d + 2) fp32 written and read back
    assert b - a == 2 * 3 * cfg.hq * (cfg.head_dim + 2) * 4


def test_decode_only_throughput_is_batch_over_the_layers_of_one_step():
    """A step decodes B tokens per rank through L decode calls (one per layer); with the
    median call time t, the decode-only throughput is world * B / (L * t), whatever the
    number of steps the samples came from."""
    calls = [0.2, 0.25, 0.3, 0.21, 0.19] * 8        # ms; 40 samples from several steps
    med, tok_s = bench.call_stats(calls, layers=32, batch=64, world=1)
    assert med == 0.21
    assert tok_s == pytest.approx(64 / (32 * 0.21e-3), rel=1e-12)
    _, tok_s2 = bench.call_stats(calls, layers=32, batch=64, world=4)
    assert tok_s2 == pytest.approx(4 * tok_s, rel=1e-12)


def test_timed_region_runs_exactly_the_requested_steps():
    for steps, per in ((20, 1), (20, 20), (20, 16), (7, 16), (200, 3), (1, 1)):
        plan = bench.chunk_plan(steps, per)
        assert sum(plan) == steps
        assert all(n == per for n in plan[:-1]) and 0 < plan[-1] <= per


class _Recorder:
    """Stand-in for the binding: records the name of every call a step makes."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args, **kw):
            self.calls.append(name)
        return call


def _runner(key, evict, select, per_step_plan=True):
    """A bench.Runner with its device state replaced by placeholders (no GPU)."""
    cfg = dataclasses.replace(W.CONFIGS[key], layers=2)
    r = object.__new__(bench.Runner)
    r.pk, r.cfg, r.L = _Recorder(), cfg, cfg.layers
    r.per_step_plan = per_step_plan
    r.incremental = bool(cfg.score) and evict == "incremental"
    r.select_in_call = r.incremental and select == "call"
    r.side = None
    r.ev_app = [None] * cfg.layers
    x = [None] * cfg.layers

    class _Wl:
        k_pool, v_pool, scale = x, x, 0.125
    r.wl = _Wl()
    r.q = r.k_new = r.v_new = r.out = r.score_pool = x
    r.bt = r.ctx = r.pos = r.err = r.ws = r.evict = r.scores = None
    r.num_splits = 0
    return r


@pytest.mark.parametrize("evict,select,per_layer", [
    ("incremental", "call", ["pa_append_kv_scored", "pa_decode_planned_select_pooled"]),
    ("incremental", "stream", ["pa_append_kv_scored", "pa_decode_planned",
                               "pe_select_evict_block_pooled"]),
    ("full", "call", ["pa_append_kv", "pa_decode_planned", "pe_score_tokens",
                      "pe_select_evict_block"]),
])
def test_c2_step_makes_each_layers_calls_once(evict, select, per_layer):
    """The c2 step: one plan, then per layer exactly the calls of its eviction mode (a
    selection inside the decode call must not bring back the full score pass)."""
    r = _runner("c2", evict, select)
    r.step()
    assert r.pk.calls == ["pa_decode_prepare"] + per_layer * r.L


class _FakeClocks:
    """Stands in for the nvidia-smi sampler: records that it ran, returns a soak record."""
    started = 0

    def __init__(self, device):
        _FakeClocks.started += 1

    def stop(self):
        return {"sm_mhz": 1700.0, "sm_max_mhz": 1965.0, "samples": 4, "reasons": ["sw_power_cap"]}


def test_clock_record_keeps_a_timed_region_with_enough_samples(monkeypatch):
    monkeypatch.setattr(bench, "Clocks", _FakeClocks)
    _FakeClocks.started = 0
    timed = {"sm_mhz": 1672.0, "sm_max_mhz": 1965.0, "samples": 7, "reasons": ["sw_power_cap"]}
    calls = []
    rec = bench.clocks_under_load(timed, "cpu", lambda: calls.append(1), timed_s=1.5)
    assert rec["sm_mhz"] == 1672.0 and rec["window"] == "timed region"
    assert calls == [] and _FakeClocks.started == 0


@pytest.mark.parametrize("timed,timed_s", [
    (None, 2.0),
    ({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "samples": 2, "reasons": []}, 2.0),
    # enough samples, but a 7 ms region: they are the idle GPU around it
    ({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "samples": 3, "reasons": []}, 0.007)])
def test_clock_record_soaks_after_a_short_timed_region(monkeypatch, timed, timed_s):
    """Fewer than 3 samples, or a region shorter than 1 s: the same step runs back to
    back for the soak time, and its samples become the record."""
    monkeypatch.setattr(bench, "Clocks", _FakeClocks)
    monkeypatch.setattr(bench.torch.cuda, "synchronize", lambda device=None: None)
    _FakeClocks.started = 0
    calls = []
    rec = bench.clocks_under_load(timed, "cpu", lambda: calls.append(1), timed_s,
                                  seconds=0.05)
    assert len(calls) >= 1 and _FakeClocks.started == 1
    assert rec["sm_mhz"] == 1700.0 and rec["reasons"] == ["sw_power_cap"]
    assert rec["timed_region"] == timed and "after the timed region" in rec["window"]
