"""CPU check of bench.py's reference arm (the fp64 oracle timed on host cores):
rank 0 prints exactly one JSON line with the keys of the benchmark line, the
reference's own cpu_baseline and an e2e entry with no host-device traffic; any
other rank does no work and prints nothing."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(workload, rank="0"):
    env = dict(os.environ, RANK=rank, WORLD_SIZE="2" if rank != "0" else "1")
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2",
                           "--warmup", "3", "--workload", workload, "--cpu-seconds", "1"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def _timed_bench(workload):
    import time
    t0 = time.perf_counter()
    r = _bench(workload)
    return r, time.perf_counter() - t0


@pytest.mark.parametrize("workload", ["c2", "p1"])
def test_reference_arm_prints_one_contract_line(workload):
    r, wall_s = _timed_bench(workload)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert (line["n_gpus"], line["steps"], line["warmup"]) == (1, 2, 3)
    assert line["higher_is_better"] is True and line["vs_baseline"] is None
    assert line["dtype"] == "f64" and line["data"] == "synthetic"
    assert isinstance(line["config"].get("workload"), str)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["unit"] == line["unit"]
    assert cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # a step is one bounded sample: the steps claimed fit in the time the run took
    assert line["steps"] * line["ms_per_step"] / 1000.0 < wall_s
    assert line["ms_per_full_step_extrapolated"] > 0


def test_reference_arm_other_ranks_do_nothing():
    r = _bench("c2", rank="1")
    assert r.returncode == 0 and r.stdout.strip() == ""
