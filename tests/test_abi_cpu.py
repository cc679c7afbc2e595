"""Host-side checks of the C-ABI library that need no GPU: it loads, it
exports every function include/*.h declares, and argument checking returns
the documented status codes before anything is enqueued."""
import ctypes
import os
import re

import pytest

from routed_expert_layer_route_b200 import build as pkg_build
from routed_expert_layer_route_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 1 << 40  # 256-byte aligned non-null pointer value; never dereferenced here


@pytest.fixture(scope="module")
def L():
    pkg_build.build()
    return moe.lib()


def declared_functions():
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(moe_[a-z0-9_]+)\s*\(", text):
            names.add(m.group(1))
    return names


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert {"moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer"} <= names
    for n in names:
        assert hasattr(L, n), n
    assert names == set(moe.SIGNATURES), names ^ set(moe.SIGNATURES)


def test_status_strings(L):
    for code in range(0, -8, -1):
        s = moe.status_string(code)
        assert s and s != "unknown status"
    assert moe.status_string(-99) == "unknown status"
    assert moe.moe_version() >= 10000


def test_workspace_size(L):
    n1 = moe.moe_workspace_size(1, 2048, 128, 768, 8)
    n2 = moe.moe_workspace_size(64, 2048, 128, 768, 8)
    assert n1 >= 256 and n2 > n1 and n1 % 256 == 0
    assert moe.moe_workspace_size(1, 100, 128, 768, 8) == 0      # d % 64
    assert moe.moe_workspace_size(1, 2048, 2000, 768, 8) == 0    # E > 1024
    assert moe.moe_workspace_size(1, 2048, 128, 770, 8) == 0     # I % 16
    assert moe.moe_workspace_size(1, 2048, 128, 768, 0) == 0     # k1 < 1
    assert moe.moe_workspace_size(1, 2048, 8, 768, 9) == 0       # k1 > E


def layer(L, T=1, d=2048, E=128, I=768, k1=8, k2=8, y=FAKE, ws=FAKE, ws_bytes=1 << 40,
          ptr=FAKE, y_dtype=1, flags=0):
    return L.moe_layer(ptr, ptr, None, ptr, ptr, ptr, T, d, E, I, k1, k2, y, y_dtype, None, None,
                       None, flags, ws, ws_bytes, None)


def test_layer_argument_checks(L):
    assert layer(L, k1=8, k2=4) == moe.MOE_ERR_INVALID_ARG           # k2 < k1
    assert layer(L, k1=0, k2=4) == moe.MOE_ERR_INVALID_ARG
    assert layer(L, E=4, k1=8, k2=8) == moe.MOE_ERR_INVALID_ARG      # k1 > E
    assert layer(L, k1=33, k2=40) == moe.MOE_ERR_INVALID_ARG          # k1 > 32
    assert layer(L, d=100) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert layer(L, I=8) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert layer(L, E=1025, k1=8) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert layer(L, y=None) == moe.MOE_ERR_INVALID_ARG
    assert layer(L, ws=None) == moe.MOE_ERR_INVALID_ARG
    assert layer(L, ws=FAKE + 16) == moe.MOE_ERR_INVALID_ARG          # ws not 256-aligned
    assert layer(L, ptr=FAKE + 8) == moe.MOE_ERR_INVALID_ARG          # misaligned tensor
    assert layer(L, y_dtype=7) == moe.MOE_ERR_INVALID_ARG
    assert layer(L, flags=9) == moe.MOE_ERR_INVALID_ARG
    assert layer(L, flags=moe.MOE_PATH_DECODE) == moe.MOE_ERR_INVALID_ARG        # needs channel-major
    assert layer(L, flags=moe.MOE_PATH_STREAM | moe.MOE_WDOWN_CHANNEL_MAJOR) == moe.MOE_ERR_INVALID_ARG
    assert layer(L, flags=0x200) == moe.MOE_ERR_INVALID_ARG
    assert layer(L, ws_bytes=1024) == moe.MOE_ERR_WORKSPACE_TOO_SMALL
    assert layer(L, T=0) == moe.MOE_OK                                 # no-op, nothing enqueued
    assert layer(L, T=0, k2=9) == moe.MOE_OK                           # k2 > E-independent, valid


def test_other_calls_argument_checks(L):
    r = L.moe_route(FAKE, FAKE, None, None, 4, 2048, 128, 8, 4, FAKE, FAKE, None, 0, None)
    assert r == moe.MOE_ERR_INVALID_ARG                                # k2 < k1
    r = L.moe_route(None, None, None, None, 4, 0, 128, 8, 16, FAKE, FAKE, None, 0, None)
    assert r == moe.MOE_ERR_INVALID_ARG                                # no logits given
    r = L.moe_route(None, None, None, FAKE, 0, 0, 128, 8, 16, FAKE, FAKE, None, 0, None)
    assert r == moe.MOE_OK                                             # T = 0
    assert L.moe_permute(FAKE, 4, 8, 2000, FAKE, FAKE, FAKE, None, 0, None) == \
        moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_permute(FAKE, 4, 8, 128, None, FAKE, FAKE, None, 0, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_expert_ffn(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2048, 128, 768, 8, FAKE, 0,
                            FAKE, 1024, None) == moe.MOE_ERR_WORKSPACE_TOO_SMALL
    assert L.moe_combine(FAKE, FAKE, FAKE, 4, 2048, 8, FAKE, 3, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_combine(FAKE, FAKE, FAKE, 4, 100, 8, FAKE, 1, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_workspace_init(None, 4096, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_pack_w_down(FAKE, FAKE, 4, 100, 32, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_pack_w_down(FAKE, FAKE, 4, 128, 32, None) == moe.MOE_ERR_INVALID_ARG  # in place
    v = ctypes.c_int(0)
    assert L.moe_read_device_status(None, ctypes.byref(v), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_test_exp_c(None, None, 0, None) == moe.MOE_OK
    # the no-alloc expert FFN refuses shapes beyond its fixed scratch before touching CUDA
    assert L.moe_expert_ffn_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 512, 64, 1024, 8, FAKE,
                                    None) == moe.MOE_ERR_SCRATCH_LIMIT
    assert L.moe_expert_ffn_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 512, 64, 1024, 8, FAKE,
                                    None) == moe.MOE_OK
    assert L.moe_expert_ffn_noalloc(FAKE, None, FAKE, FAKE, FAKE, FAKE, 4, 512, 64, 1024, 8, FAKE,
                                    None) == moe.MOE_ERR_INVALID_ARG


def test_cascade_argument_checks(L):
    nan = float("nan")
    r = L.moe_route_cascade(None, None, None, FAKE, 4, 0, 128, 8, 16, nan, FAKE, FAKE, None, None,
                            0, None)
    assert r == moe.MOE_ERR_INVALID_ARG                                # tau NaN
    r = L.moe_route_cascade(None, None, None, FAKE, 4, 0, 128, 8, 4, 0.5, FAKE, FAKE, None, None, 0,
                            None)
    assert r == moe.MOE_ERR_INVALID_ARG                                # k2 < k1
    r = L.moe_route_cascade(None, None, None, FAKE, 0, 0, 128, 8, 16, 0.9, FAKE, FAKE, None, None,
                            0, None)
    assert r == moe.MOE_OK                                             # T = 0

    def lc(tau=0.7, k1=8, k2=8, T=1):
        return L.moe_layer_cascade(FAKE, FAKE, None, FAKE, FAKE, FAKE, T, 2048, 128, 768, k1, k2,
                                   tau, FAKE, 1, None, None, None, None, 0, FAKE, 1 << 40, None)
    assert lc(tau=nan) == moe.MOE_ERR_INVALID_ARG
    assert lc(k1=8, k2=4) == moe.MOE_ERR_INVALID_ARG
    assert lc(T=0) == moe.MOE_OK


def test_binding_raises_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        moe.lib()


def test_skip_argument_checks(L):
    nan, inf = float("nan"), float("inf")

    def rs(tab=FAKE, th_e=0.5, th_w=0.1, k1=8, k2=16, T=4):
        return L.moe_route_skip(None, None, None, FAKE, T, 0, 128, k1, k2, tab, th_e, th_w, FAKE,
                                FAKE, None, None, 0, None)
    assert rs(tab=None) == moe.MOE_ERR_INVALID_ARG                      # no table
    assert rs(th_e=nan) == moe.MOE_ERR_INVALID_ARG
    assert rs(th_w=nan) == moe.MOE_ERR_INVALID_ARG
    assert rs(k1=8, k2=4) == moe.MOE_ERR_INVALID_ARG                    # k2 < k1
    assert rs(th_w=inf, T=0) == moe.MOE_OK                              # T = 0, infinite threshold

    def ls(tab=FAKE, th_e=0.5, th_w=0.1, T=1):
        return L.moe_layer_skip(FAKE, FAKE, None, FAKE, FAKE, FAKE, T, 2048, 128, 768, 8, 8, tab,
                                th_e, th_w, FAKE, 1, None, None, None, None, 0, FAKE, 1 << 40, None)
    assert ls(tab=None) == moe.MOE_ERR_INVALID_ARG
    assert ls(th_e=nan) == moe.MOE_ERR_INVALID_ARG
    assert ls(T=0) == moe.MOE_OK


def test_channel_topk_argument_checks(L):
    def lc(keep=100, k1=8, k2=8, I=768, T=1, y_dtype=1, norms=FAKE):
        return L.moe_layer_channel_topk(FAKE, FAKE, None, FAKE, FAKE, FAKE, norms, T, 2048, 128, I,
                                        k1, k2, keep, FAKE, y_dtype, None, None, None, None, None,
                                        None, FAKE, 1 << 40, None)
    assert lc(keep=0) == moe.MOE_ERR_INVALID_ARG
    assert lc(keep=8 * 768 + 1) == moe.MOE_ERR_INVALID_ARG               # more than k1*I
    assert lc(y_dtype=7) == moe.MOE_ERR_INVALID_ARG
    assert lc(k1=8, k2=4) == moe.MOE_ERR_INVALID_ARG
    assert lc(I=4096, keep=100) == moe.MOE_ERR_UNSUPPORTED_SHAPE         # 8*4096 channels > 16384
    assert lc(T=0) == moe.MOE_OK
    assert lc(norms=None) == moe.MOE_ERR_INVALID_ARG
    r = L.moe_channel_norms(FAKE, 128, 2048, 770, 0, FAKE, None)         # I % 16 != 0
    assert r == moe.MOE_ERR_UNSUPPORTED_SHAPE
    r = L.moe_channel_norms(FAKE, 128, 2048, 768, 0x7, FAKE, None)       # unknown flag
    assert r == moe.MOE_ERR_INVALID_ARG


def test_headers_are_plain_c(tmp_path):
    # the boundary is a C ABI: both headers compile as strict C99, no C++ or CUDA types
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_headers.c"
    src.write_text('#include "moe.h"\n#include "moe_testing.h"\nint main(void) { return 0; }\n')
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    r = subprocess.run([gcc, "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                        "-fsyntax-only", "-I", inc, str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
