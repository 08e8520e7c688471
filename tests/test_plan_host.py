"""CPU test of the host-side decode launch plan (no GPU needed).

Compiles a small host program against libpagedkv.so that prints the plan the
library makes for a list of shapes, and checks its invariants: which kernel
runs, that the pipeline fits in shared memory with at least two stages of
about 64 KB, that the workspace covers every partition slot, and that the
partition slots cover the longest context."""
import os
import subprocess
import tempfile

import pytest

from paged_kv_cache_396_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "paged_kv_cache_396_b200")

# name, B, Hq, Hkv, d, bs, MB, kv (0 bf16, 1 INT8, 2 FP8), num_splits, staged?
CASES = [
    ("c1", 2, 4, 2, 64, 16, 7, 0, 0, 1),
    ("c2", 32, 32, 8, 64, 16, 65, 0, 0, 1),
    ("c3", 64, 32, 8, 128, 16, 513, 0, 0, 1),
    ("c4", 4, 32, 8, 128, 256, 512, 0, 0, 1),
    ("c5", 128, 64, 8, 128, 16, 257, 1, 0, 1),
    ("g16", 3, 64, 4, 64, 16, 32, 0, 0, 1),
    ("i8g16", 3, 64, 4, 128, 16, 19, 1, 0, 1),
    ("mqa", 8, 16, 1, 128, 32, 40, 0, 0, 1),
    ("split1", 3, 32, 8, 128, 16, 126, 0, 1, 1),
    ("split8", 3, 32, 8, 128, 16, 126, 0, 8, 1),
    ("bs12", 4, 64, 4, 128, 12, 60, 0, 0, 0),
    ("i8d64", 3, 64, 8, 64, 16, 13, 1, 0, 0),
    ("hkv16", 2, 32, 16, 64, 16, 10, 0, 0, 0),
    ("f8", 128, 64, 8, 128, 16, 257, 2, 0, 1),
    ("f8g16", 3, 64, 4, 128, 16, 19, 2, 0, 1),
    ("f8split96", 3, 64, 8, 128, 16, 126, 2, 96, 1),
    ("f8d64", 3, 64, 8, 64, 16, 13, 2, 0, 0),
]

PROBE = r"""
#include <cstdio>
#include <cstdlib>
#include "kernels.h"
int main(int argc, char **argv) {
    int B = atoi(argv[1]), Hq = atoi(argv[2]), Hkv = atoi(argv[3]), d = atoi(argv[4]);
    int bs = atoi(argv[5]), MB = atoi(argv[6]), kv = atoi(argv[7]), ns = atoi(argv[8]);
    pkv::DecodePlan p = pkv::make_decode_plan(B, Hq, Hkv, d, bs, MB, ns, kv, 148);
    printf("%d %d %d %d %d %d %d %d %d %d %d %d %zu %zu %zu\n", p.kernel, p.S, p.chunk, p.wph,
           p.tpw, p.n_sub, p.nstage, p.stage_bytes, p.smem_bytes, p.v_off, p.ks_off, p.vs_off,
           p.off_ml, p.off_acc, p.ws_total);
    return 0;
}
"""


@pytest.fixture(scope="module")
def probe():
    build_lib.build()
    d = tempfile.mkdtemp(prefix="pkv_plan_")
    src = os.path.join(d, "probe.cu")
    exe = os.path.join(d, "probe")
    open(src, "w").write(PROBE)
    subprocess.run([build_lib.NVCC, "-std=c++17", "-Wno-deprecated-gpu-targets", "-I",
                    os.path.join(ROOT, "include"), "-I", os.path.join(PKG, "csrc"), src, "-o", exe,
                    "-L", PKG, "-lpagedkv", "-Xlinker", f"-rpath={PKG}"], check=True,
                   capture_output=True)

    def run(*args):
        out = subprocess.run([exe, *map(str, args)], check=True, capture_output=True, text=True)
        v = out.stdout.split()
        keys = ["kernel", "S", "chunk", "wph", "tpw", "n_sub", "nstage", "stage_bytes",
                "smem_bytes", "v_off", "ks_off", "vs_off", "off_ml", "off_acc", "ws_total"]
        return dict(zip(keys, map(int, v)))
    return run


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_plan_invariants(probe, case):
    name, B, Hq, Hkv, d, bs, MB, kv_kind, ns, staged = case
    p = probe(B, Hq, Hkv, d, bs, MB, kv_kind, ns)
    i8 = kv_kind == 1
    assert p["kernel"] == staged
    max_ctx = MB * bs
    assert p["S"] * p["chunk"] >= max_ctx            # partitions cover the longest context
    if ns > 0:
        assert p["S"] <= ns
    if not staged:
        return
    assert p["chunk"] % 16 == 0 and p["chunk"] >= 16
    assert p["wph"] * Hkv == 8 and p["n_sub"] == p["wph"] * p["tpw"] and p["n_sub"] <= 32
    assert 2 <= p["nstage"] <= 8
    assert p["smem_bytes"] <= 227 * 1024
    assert p["stage_bytes"] % 1024 == 0 and p["stage_bytes"] <= 68 * 1024
    # K and V regions of n_sub sub-tiles of 16 tokens x Hkv x d elements, then scales
    elt = 1 if kv_kind else 2
    kv = p["n_sub"] * 16 * Hkv * d * elt
    assert p["v_off"] == kv and p["ks_off"] == 2 * kv
    assert p["vs_off"] - p["ks_off"] == (p["n_sub"] * 16 * Hkv * 4 if i8 else 0)
    assert 2 * kv >= 32 * 1024                       # stages are not tiny
    slots = B * p["S"] * p["wph"] * Hq
    assert p["off_acc"] - p["off_ml"] >= slots * 2 * 4
    assert p["ws_total"] - p["off_acc"] >= slots * d * 4


def test_plan_is_deterministic_and_monotone_in_splits(probe):
    a = probe(64, 32, 8, 128, 16, 513, 0, 4)
    b = probe(64, 32, 8, 128, 16, 513, 0, 4)
    assert a == b
    sizes = [probe(64, 32, 8, 128, 16, 513, 0, n)["ws_total"] for n in (1, 2, 4, 8, 16)]
    assert sizes == sorted(sizes)
