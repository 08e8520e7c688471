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


def test_product_path_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "paged_kv_cache_396_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle", text, flags=re.M), f
                assert "liboracle" not in text, f
