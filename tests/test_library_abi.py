"""CPU checks of the C ABI: the library builds and loads, exports every function
include/pagedkv.h declares, and rejects bad arguments on the host (these paths
return before any CUDA call, so they run without a GPU)."""
import ctypes
import os
import re

import pytest

from paged_kv_cache_396_b200 import build_lib
from paged_kv_cache_396_b200 import pagedkv as pk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return pk.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("pa_append_kv", "pa_decode", "pe_score_tokens", "pe_select_evict_block",
              "pa_append_kv_int8", "pa_decode_int8", "pa_decode_workspace_bytes",
              "pa_status_string"):
        assert n in names
    assert set(pk.EXPORTED) <= set(names)


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in pagedkv.h but not exported"
    assert lib.pa_version().startswith(b"pagedkv")
    assert lib.pa_status_string(0) == b"ok"
    assert b"NULL" in lib.pa_status_string(-1)


FAKE = ctypes.c_void_p(1 << 20)       # 16-byte aligned, never dereferenced
ODD = ctypes.c_void_p((1 << 20) + 2)  # misaligned


def _decode(lib, **kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, stride=16 * 8 * 128, bt=FAKE, MB=4, ctx=FAKE, B=2,
             Hq=32, Hkv=8, d=128, bs=16, N=10, scale=0.1, S=0, ws=None, wsb=0, err=FAKE)
    a.update(kw)
    return lib.pa_decode(a["out"], a["q"], a["k"], a["v"], a["stride"], a["bt"], a["MB"],
                         a["ctx"], a["B"], a["Hq"], a["Hkv"], a["d"], a["bs"], a["N"], a["scale"],
                         a["S"], a["ws"], a["wsb"], a["err"], None)


def test_decode_rejects_bad_arguments_on_host(lib):
    assert _decode(lib, q=None) == -1
    assert _decode(lib, err=None) == -1
    assert _decode(lib, Hq=30) == -2            # Hq % Hkv != 0
    assert _decode(lib, Hq=8 * 17) == -2        # G > 16
    assert _decode(lib, d=96) == -2             # unsupported head_dim
    assert _decode(lib, stride=100) == -2       # block stride smaller than a block
    assert _decode(lib, bs=0) == -2
    assert _decode(lib, B=-1) == -2
    assert _decode(lib, scale=float("nan")) == -2
    assert _decode(lib, k=ODD) == -3
    assert _decode(lib, stride=16 * 8 * 128 + 4) == -3  # stride not a multiple of 16 bytes
    assert _decode(lib, B=0) == 0               # empty batch: nothing to do
    # the documented maximum sizes
    assert _decode(lib, B=65536) == -2
    assert _decode(lib, Hq=65536 * 2, Hkv=65536) == -2
    assert _decode(lib, N=1 << 31) == -2
    assert _decode(lib, MB=(1 << 27) + 1, bs=16) == -2   # MB*bs > 2^31 - 1
    # the largest accepted sizes pass the shape checks and stop at the missing workspace
    # (-4) on a GPU machine, or at the device query (-5 / -6) without one: never a launch
    assert _decode(lib, B=65535, MB=(1 << 27) - 1) in (-4, -5, -6)


def test_append_and_score_reject_bad_arguments_on_host(lib):
    assert lib.pa_append_kv(FAKE, FAKE, FAKE, FAKE, 2048, FAKE, 4, FAKE, 2, 1, 8, 128, 16, 10,
                            None, None, None) == -1
    assert lib.pa_append_kv(FAKE, FAKE, FAKE, FAKE, 2048, FAKE, 4, FAKE, 2, -1, 8, 128, 16, 10,
                            None, FAKE, None) == -2
    assert lib.pa_append_kv(ODD, FAKE, FAKE, FAKE, 16 * 8 * 128, FAKE, 4, FAKE, 2, 1, 8, 128, 16,
                            10, None, FAKE, None) == -3
    assert lib.pa_append_kv_int8(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16 * 8 * 128 + 8, FAKE, 4,
                                 FAKE, 2, 1, 8, 128, 16, 10, None, FAKE, None) == -3
    assert lib.pe_score_tokens(FAKE, FAKE, FAKE, 2048, FAKE, 4, FAKE, 2, 8, 128, 16, 10, None,
                               None) == -1
    assert lib.pe_score_tokens(FAKE, FAKE, FAKE, 2048, FAKE, 4, FAKE, 2, 8, 32, 16, 10, FAKE,
                               None) == -2
    assert lib.pe_select_evict_block(None, None, FAKE, FAKE, 2, 4, 8, 16, None) == -1
    assert lib.pe_select_evict_block(FAKE, None, FAKE, FAKE, 2, 0, 8, 16, None) == -2
    assert lib.pe_select_evict_block(FAKE, None, FAKE, FAKE, 0, 4, 8, 16, None) == 0


NUL = None
S = 16 * 8 * 128   # dense block stride of a [bs=16][Hkv=8][d=128] block


def _dec(fn, lib, *, kv="bf16", **kw):
    """pa_decode_int8 / pa_decode_fp8 / pa_decode_static_scratch with one argument changed."""
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, ks=FAKE, vs=FAKE, stride=S, bt=FAKE, MB=4,
             ctx=FAKE, B=2, Hq=32, Hkv=8, d=128, bs=16, N=10, scale=0.1, S=0, err=FAKE,
             ev=FAKE, sp=FAKE)
    a.update(kw)
    common = (a["stride"], a["bt"], a["MB"], a["ctx"], a["B"], a["Hq"], a["Hkv"], a["d"], a["bs"],
              a["N"], a["scale"], a["S"])
    if fn == "int8":
        return lib.pa_decode_int8(a["out"], a["q"], a["k"], a["v"], a["ks"], a["vs"], *common,
                                  None, 0, a["err"], None)
    if fn == "fp8":
        return lib.pa_decode_fp8(a["out"], a["q"], a["k"], a["v"], *common, None, 0, a["err"],
                                 None)
    if fn == "planned":
        return lib.pa_decode_planned(a["out"], a["q"], a["k"], a["v"], *common, None, 0,
                                     a["err"], None)
    if fn == "int8_planned":
        return lib.pa_decode_int8_planned(a["out"], a["q"], a["k"], a["v"], a["ks"], a["vs"],
                                          *common, None, 0, a["err"], None)
    if fn in ("select", "planned_select"):
        f = lib.pa_decode_select_pooled if fn == "select" else lib.pa_decode_planned_select_pooled
        return f(a["out"], a["q"], a["k"], a["v"], *common, None, 0, a["ev"], None, a["sp"],
                 a["err"], None)
    if fn == "fp8_planned":
        return lib.pa_decode_fp8_planned(a["out"], a["q"], a["k"], a["v"], *common, None, 0,
                                         a["err"], None)
    return lib.pa_decode_static_scratch(a["out"], a["q"], a["k"], a["v"], *common, a["err"], None)


def test_decode_variants_reject_bad_arguments_on_host(lib):
    for fn in ("int8", "fp8", "static", "planned", "int8_planned", "fp8_planned", "select",
               "planned_select"):
        assert _dec(fn, lib, q=NUL) == -1, fn
        assert _dec(fn, lib, err=NUL) == -1, fn
        assert _dec(fn, lib, Hq=24, Hkv=16) == -2, fn      # Hq % Hkv != 0
        assert _dec(fn, lib, Hq=8 * 32) == -2, fn          # G > 16
        assert _dec(fn, lib, d=80) == -2, fn
        assert _dec(fn, lib, stride=S - 16) == -2, fn      # block stride below one block
        assert _dec(fn, lib, scale=float("nan")) == -2, fn
        assert _dec(fn, lib, out=ODD) == -3, fn
        assert _dec(fn, lib, B=0) == 0, fn
    assert _dec("int8", lib, ks=NUL) == -1
    assert _dec("int8", lib, vs=NUL) == -1
    assert _dec("int8", lib, ks=ODD) == -3                 # scale pools: 16-byte aligned
    assert _dec("int8", lib, vs=ctypes.c_void_p((1 << 20) + 4)) == -3
    assert _dec("int8", lib, stride=S + 8) == -3           # one-byte pool: 8 B not a multiple
    assert _dec("fp8", lib, stride=S + 8) == -3
    assert _dec("static", lib, S=-1) == -2
    assert _dec("static", lib, stride=S + 4) == -3         # bf16: 8 bytes
    assert _dec("int8_planned", lib, ks=NUL) == -1
    assert _dec("planned", lib, stride=S + 4) == -3
    for fn in ("select", "planned_select"):          # the selection's own outputs and input
        assert _dec(fn, lib, ev=NUL) == -1, fn
        assert _dec(fn, lib, sp=NUL) == -1, fn
        assert _dec(fn, lib, ev=NUL, B=0) == 0, fn


def test_decode_prepare_rejects_bad_arguments_on_host(lib):
    def prep(**kw):
        a = dict(ctx=FAKE, B=2, Hq=32, Hkv=8, d=128, bs=16, MB=4, S=0, ws=None, wsb=0, err=FAKE)
        a.update(kw)
        return lib.pa_decode_prepare(a["ctx"], a["B"], a["Hq"], a["Hkv"], a["d"], a["bs"],
                                     a["MB"], a["S"], a["ws"], a["wsb"], a["err"], None)
    assert prep(ctx=NUL) == -1
    assert prep(err=NUL) == -1
    assert prep(B=-1) == -2
    assert prep(B=65536) == -2
    assert prep(Hq=30) == -2
    assert prep(Hq=8 * 17) == -2
    assert prep(d=96) == -2
    assert prep(bs=0) == -2
    assert prep(MB=(1 << 27) + 1) == -2
    assert prep(B=0) == 0
    # valid sizes stop at the missing workspace on a GPU machine, or at the device query
    # without one: never a launch
    assert prep() in (-4, -5, -6)


def test_appends_reject_bad_arguments_on_host(lib):
    def fp8(**kw):
        a = dict(kn=FAKE, vn=FAKE, k=FAKE, v=FAKE, stride=S, bt=FAKE, MB=4, pos=FAKE, B=2, n=1,
                 Hkv=8, d=128, bs=16, N=10, slots=None, err=FAKE)
        a.update(kw)
        return lib.pa_append_kv_fp8(*a.values(), None)

    assert fp8(B=0) == 0 and fp8(n=0) == 0
    assert fp8(k=NUL) == -1 and fp8(err=NUL) == -1
    assert fp8(n=-2) == -2 and fp8(d=32) == -2 and fp8(bs=0) == -2 and fp8(N=0) == -2
    assert fp8(stride=S - 1) == -2
    assert fp8(kn=ODD) == -3 and fp8(stride=S + 8) == -3

    def scored(**kw):
        a = dict(kn=FAKE, vn=FAKE, k=FAKE, v=FAKE, stride=S, pool=FAKE, bt=FAKE, MB=4, pos=FAKE,
                 B=2, n=1, Hkv=8, d=128, bs=16, N=10, slots=None, err=FAKE)
        a.update(kw)
        return lib.pa_append_kv_scored(*a.values(), None)

    assert scored(pool=NUL) == -1 and scored(n=-1) == -2 and scored(v=ODD) == -3
    assert scored(B=0, pool=NUL) == 0

    def i8scored(**kw):
        a = dict(kn=FAKE, vn=FAKE, kq=FAKE, vq=FAKE, ks=FAKE, vs=FAKE, pool=FAKE, stride=S,
                 bt=FAKE, MB=4, pos=FAKE, B=2, n=1, Hkv=8, d=128, bs=16, N=10, slots=None,
                 err=FAKE)
        a.update(kw)
        return lib.pa_append_kv_int8_scored(*a.values(), None)

    assert i8scored(pool=NUL) == -1 and i8scored(ks=NUL) == -1
    assert i8scored(vs=ODD) == -3 and i8scored(stride=S + 8) == -3
    assert i8scored(Hkv=0) == -2


def test_eviction_calls_reject_bad_arguments_on_host(lib):
    # pooled select: evict, means, score_pool, bt, MB, ctx, B, Hkv, bs, N, err, stream
    assert lib.pe_select_evict_block_pooled(FAKE, None, FAKE, FAKE, 4, FAKE, 0, 8, 16, 10, NUL,
                                            None) == 0
    assert lib.pe_select_evict_block_pooled(FAKE, None, NUL, FAKE, 4, FAKE, 2, 8, 16, 10, FAKE,
                                            None) == -1
    assert lib.pe_select_evict_block_pooled(FAKE, None, FAKE, FAKE, 0, FAKE, 2, 8, 16, 10, FAKE,
                                            None) == -2
    assert lib.pe_select_evict_block_pooled(FAKE, None, FAKE, FAKE, 4, FAKE, 70000, 8, 16, 10,
                                            FAKE, None) == -2
    # compaction: bt, MB, ctx, freed, evict|mask, B, bs, err, stream
    for f in (lib.pe_evict_compact, lib.pe_evict_compact_mask):
        assert f(FAKE, 4, FAKE, None, FAKE, 0, 16, NUL, None) == 0
        assert f(NUL, 4, FAKE, None, FAKE, 2, 16, FAKE, None) == -1
        assert f(FAKE, 4, FAKE, None, NUL, 2, 16, FAKE, None) == -1
        assert f(FAKE, 4, FAKE, None, FAKE, 2, 16, NUL, None) == -1
        assert f(FAKE, 0, FAKE, None, FAKE, 2, 16, FAKE, None) == -2
        assert f(FAKE, 4, FAKE, None, FAKE, 2, 0, FAKE, None) == -2
        assert f(FAKE, 1 << 20, FAKE, None, FAKE, 2, 1 << 12, FAKE, None) == -2  # MB*bs > 2^31
    # threshold: mask, count, means, scores, ctx, B, MB, Hkv, bs, used, total, ratio, thr, stream

    def thr(**kw):
        a = dict(mask=FAKE, count=FAKE, means=None, scores=FAKE, ctx=FAKE, B=2, MB=4, Hkv=8,
                 bs=16, used=90, total=100, ratio=0.2, thr=0.5)
        a.update(kw)
        return lib.pe_select_evict_threshold(*a.values(), None)

    assert thr(B=0, mask=NUL) == 0
    assert thr(mask=NUL) == -1 and thr(count=NUL) == -1 and thr(scores=NUL) == -1
    assert thr(ratio=1.5) == -2 and thr(ratio=-0.1) == -2 and thr(ratio=float("nan")) == -2
    assert thr(thr=float("nan")) == -2 and thr(used=-1) == -2 and thr(total=-1) == -2
    assert thr(MB=0) == -2 and thr(Hkv=0) == -2 and thr(bs=0) == -2


def test_prefill_stage_rejects_bad_arguments_on_host(lib):
    # scores: scores, k, v, T, Hkv, d, stream
    assert lib.pe_prefill_scores(NUL, NUL, NUL, 0, 8, 128, None) == 0
    assert lib.pe_prefill_scores(NUL, FAKE, FAKE, 64, 8, 128, None) == -1
    assert lib.pe_prefill_scores(FAKE, NUL, FAKE, 64, 8, 128, None) == -1
    assert lib.pe_prefill_scores(FAKE, FAKE, FAKE, 64, 8, 96, None) == -2
    assert lib.pe_prefill_scores(FAKE, FAKE, FAKE, -1, 8, 128, None) == -2
    assert lib.pe_prefill_scores(FAKE, FAKE, FAKE, 64, 0, 128, None) == -2
    assert lib.pe_prefill_scores(FAKE, ODD, FAKE, 64, 8, 128, None) == -3
    # select: keep, kept, scores, cu, B, budget, err, stream
    assert lib.pe_prefill_select(NUL, NUL, NUL, NUL, 0, 16, NUL, None) == 0
    assert lib.pe_prefill_select(FAKE, FAKE, FAKE, FAKE, 2, 16, NUL, None) == -1
    assert lib.pe_prefill_select(FAKE, FAKE, FAKE, FAKE, 2, 0, FAKE, None) == -2
    assert lib.pe_prefill_select(FAKE, FAKE, FAKE, FAKE, -3, 16, FAKE, None) == -2

    # pack: k_cache, v_cache, stride, bt, MB, k, v, cu, keep, kept, B, budget, Hkv, d, bs, N, err
    def pack(**kw):
        a = dict(kc=FAKE, vc=FAKE, stride=S, bt=FAKE, MB=4, k=FAKE, v=FAKE, cu=FAKE, keep=FAKE,
                 kept=FAKE, B=2, budget=64, Hkv=8, d=128, bs=16, N=10, err=FAKE)
        a.update(kw)
        return lib.pe_prefill_pack(*a.values(), None)

    assert pack(B=0, kc=NUL) == 0
    assert pack(kc=NUL) == -1 and pack(keep=NUL) == -1 and pack(k=NUL) == -1
    assert pack(budget=0) == -2 and pack(stride=S - 8) == -2 and pack(d=48) == -2
    assert pack(kc=ODD) == -3 and pack(k=ODD) == -3 and pack(stride=S + 4) == -3

    # compress: k_cache, v_cache, stride, bt, MB, k, v, cu, T, B, budget, Hkv, d, bs, N,
    #           scores, keep, kept, err
    def compress(**kw):
        a = dict(kc=FAKE, vc=FAKE, stride=S, bt=FAKE, MB=4, k=FAKE, v=FAKE, cu=FAKE, T=100, B=2,
                 budget=64, Hkv=8, d=128, bs=16, N=10, scores=FAKE, keep=FAKE, kept=FAKE,
                 err=FAKE)
        a.update(kw)
        return lib.pe_prefill_compress(*a.values(), None)

    assert compress(B=0, kc=NUL) == 0
    assert compress(scores=NUL) == -1 and compress(err=NUL) == -1 and compress(v=NUL) == -1
    assert compress(T=-5) == -2 and compress(budget=0) == -2 and compress(stride=100) == -2
    assert compress(vc=ODD) == -3 and compress(v=ODD) == -3


def test_prefill_attention_rejects_bad_arguments_on_host(lib):
    # out, q, cu_q, max_q_len, k, v, stride, bt, MB, ctx, B, Hq, Hkv, d, bs, N, scale, err,
    # workspace, workspace_bytes, stream
    def attn(**kw):
        a = dict(out=FAKE, q=FAKE, cu=FAKE, mq=512, k=FAKE, v=FAKE, stride=S, bt=FAKE, MB=4,
                 ctx=FAKE, B=2, Hq=32, Hkv=8, d=128, bs=16, N=10, scale=0.1, err=FAKE, ws=None,
                 wsb=0)
        a.update(kw)
        return lib.pa_prefill_attention(*a.values(), None)

    assert attn(B=0, q=NUL) == 0 and attn(mq=0, q=NUL) == 0
    assert attn(q=NUL) == -1 and attn(cu=NUL) == -1 and attn(err=NUL) == -1
    assert attn(Hq=24) == -2                      # G = 3: not a power of two
    assert attn(Hq=8 * 32) == -2                  # G = 32
    assert attn(Hq=4) == -2                       # Hq < Hkv
    assert attn(d=256) == -2 and attn(mq=-1) == -2 and attn(scale=float("nan")) == -2
    assert attn(stride=S - 128) == -2
    assert attn(q=ODD) == -3 and attn(stride=S + 4) == -3
    assert attn(ws=ODD, wsb=4096) == -3           # workspace: 16-byte aligned
    assert lib.pa_prefill_attention_workspace_bytes(2, 24, 8, 128, 16, 512) == 0   # G = 3
    assert lib.pa_prefill_attention_workspace_bytes(0, 32, 8, 128, 16, 512) == 0


def test_plan_and_selftest_reject_bad_arguments_on_host(lib):
    o = (ctypes.c_int * 4)()
    p = ctypes.cast(o, ctypes.c_void_p)
    assert lib.pa_decode_plan(2, 32, 8, 128, 16, 4, 0, None, p, None, None) == -1
    assert lib.pa_decode_plan(2, 32, 8, 96, 16, 4, 0, p, p, None, None) == -2
    assert lib.pa_decode_plan(-1, 32, 8, 128, 16, 4, 0, p, p, None, None) == -2
    assert lib.pa_decode_plan(2, 32, 8, 128, 0, 4, 0, p, p, None, None) == -2
    assert lib.pa_decode_workspace_bytes(0, 32, 8, 128, 16, 4, 0) == 0
    assert lib.pa_selftest_wait_timeout(None, None) == -1


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "pagedkv.h"
int main(void) {
    /* host-side paths only: no device memory is touched */
    char *fake = (char *)(uintptr_t)(1u << 20);  /* aligned, never dereferenced */
    int rc_null = pa_decode(NULL, NULL, NULL, NULL, 2048, NULL, 4, NULL, 2, 32, 8, 128, 16, 10,
                            0.1f, 0, NULL, 0, NULL, NULL);
    int rc_shape = pe_select_evict_block((int32_t *)fake, NULL, (const float *)fake,
                                         (const int32_t *)fake, 2, 0, 8, 16, NULL);
    int rc_empty = pa_append_kv(NULL, NULL, NULL, NULL, 2048, NULL, 4, NULL, 0, 1, 8, 128, 16, 10,
                                NULL, NULL, NULL);
    printf("%s|%d|%d|%d|%s\n", pa_version(), rc_null, rc_shape, rc_empty,
           pa_status_string(PA_ERR_ALIGN));
    return strncmp(pa_version(), "pagedkv", 7) != 0;
}
"""


def test_plain_c_client_links_and_calls_the_library(lib, tmp_path):
    """The boundary is usable from C alone: a C99 program built against
    include/pagedkv.h links libpagedkv.so and gets the documented host status codes;
    the header also compiles as C++."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None or shutil.which("g++") is None:
        pytest.skip("no host C compiler")
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    libdir = os.path.dirname(build_lib.build())
    exe = tmp_path / "client"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I",
                    os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir,
                    "-lpagedkv", "-Wl,-rpath," + libdir], check=True)
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x",
                    "c++", "-I", os.path.join(ROOT, "include"), str(src)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.strip()
    version, rc_null, rc_shape, rc_empty, align_text = out.split("|")
    assert version == lib.pa_version().decode()
    assert (int(rc_null), int(rc_shape), int(rc_empty)) == (-1, -2, 0)
    assert align_text == lib.pa_status_string(-3).decode()


def test_product_path_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "paged_kv_cache_396_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle", text, flags=re.M), f
                assert "liboracle" not in text, f
