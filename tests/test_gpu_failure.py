"""The device failure path without a GPU fault: a bounded pipeline wait on a phase
nothing completes gives up after ~2 s, the kernel reports PA_DEV_TIMEOUT through the
error flag and returns, and the same CUDA context then runs a decode that matches
the oracle."""
import time

import pytest
import torch

from helpers import Device, assert_attention_close, oracle_step
from paged_kv_cache_396_b200 import pagedkv as pk
from paged_kv_cache_396_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_stays_usable():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    pk.pa_selftest_wait_timeout(err)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert err.item() == pk.PA_DEV_TIMEOUT
    assert 1.0 < dt < 30.0
    # the context is intact: a decode step right after matches the oracle
    wl = W.generate(W.CONFIGS["c1"], "cpu")
    ref = oracle_step(wl, 0, range(wl.cfg.batch))
    dev = Device(wl)
    dev.step(0)
    torch.cuda.synchronize()
    assert dev.err.item() == 0
    assert_attention_close(dev.out[0], ref["out"], "decode after the timeout self-test")
