"""The C-ABI library: it loads without a GPU, exports every symbol of include/llmint8.h, and
its host-only entry points behave (workspace sizes, status strings).  No compute calls."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

from int8_quantized_02_b200 import build as build_mod
from int8_quantized_02_b200 import llmint8

HEADER = os.path.join(build_mod.ROOT, "include", "llmint8.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return llmint8.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(llmint8_\w+)\s*\(", src)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("llmint8_quantize_weight_colwise", "llmint8_quantize_rows_and_find_outliers",
              "llmint8_linear", "llmint8_dequant"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", llmint8.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(lib, n)
    # the binding declares a prototype for each of them, and nothing else
    assert sorted(llmint8.PROTOTYPES) == names


def test_only_the_c_abi_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", llmint8.library_path()],
                         capture_output=True, text=True, check=True).stdout
    ours = set(re.findall(r"\bT (\w+)", out))
    assert ours == set(declared_functions())


def test_status_strings(lib):
    for code in range(8):
        s = llmint8.status_string(code)
        assert s and s != "unknown status"
    assert llmint8.status_string(99) == "unknown status"


def test_release_and_debug_builds_export_the_same_abi(lib):
    # the release library reports no debug checks; the debug build (LLMINT8_DEBUG) reports
    # them and exports exactly the same symbols
    assert llmint8.build_flags() & 1 == 0
    path = build_mod.build(debug=True)
    dbg = ctypes.CDLL(path)
    dbg.llmint8_build_flags.restype = ctypes.c_int
    assert dbg.llmint8_build_flags() & 1 == 1
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    assert set(re.findall(r"\bT (\w+)", out)) == set(declared_functions())
    dbg.llmint8_status_string.restype = ctypes.c_char_p
    assert b"debug" in dbg.llmint8_status_string(llmint8.ERR_DEVICE_CHECK)


def test_workspace_sizes(lib):
    f = llmint8.llmint8_linear_workspace_size
    base = f(16, 1024, 1024, 0)
    assert base > 16 * 1024          # holds at least Xq
    assert f(16, 1024, 1024, 64) > base
    assert f(32, 1024, 1024, 64) > f(17, 1024, 1024, 64)
    # shapes outside the rules give 0
    assert f(0, 1024, 1024, 0) == 0
    assert f(16, 1000, 1024, 0) == 0          # N not a multiple of 16
    assert f(16, 1024, 1000, 0) == 0          # K not a multiple of 16
    assert f(16, 1024, 262144, 0) == 0        # K too large for int32 accumulation
    assert f(16, 1024, 1024, 2048) == 0       # capacity above K
    assert f(16, 1024, 1024, -1) == 0
    q = llmint8.llmint8_quantize_workspace_size
    assert q(16, 1024) >= 256 and q(0, 1024) == 0
    assert q(4096, 16384) % 256 == 0


def test_default_capacity():
    assert llmint8.default_max_outliers(4096, 6.0) == 512
    assert llmint8.default_max_outliers(4096, 0.0) == 4096
    assert llmint8.default_max_outliers(64, 6.0) == 64


def test_wait_timeout_setter(lib):
    assert lib.llmint8_set_wait_timeout_ns(ctypes.c_uint64(5)) == 0
    assert lib.llmint8_set_wait_timeout_ns(ctypes.c_uint64(0)) == 0   # restores the default


def test_next_bitmaps_arguments_are_checked_before_any_launch(lib):
    # a missing or misaligned bitmap output, or a NaN next threshold, is rejected on the host
    fake = ctypes.c_void_p(1 << 20)     # aligned, never dereferenced: the checks come first
    args = lambda nt, bits: (fake, 64, 1024, fake, fake, 1024, None, None,  # noqa: E731
                             ctypes.c_float(6.0), 64, fake, fake, 1 << 30, None, None,
                             ctypes.c_float(nt), bits)
    assert lib.llmint8_linear_next_bitmaps(*args(6.0, None)) == llmint8.ERR_INVALID_ARG
    assert lib.llmint8_linear_next_bitmaps(*args(6.0, ctypes.c_void_p((1 << 20) + 2))) == \
        llmint8.ERR_INVALID_ARG
    assert lib.llmint8_linear_next_bitmaps(*args(float("nan"), fake)) == \
        llmint8.ERR_INVALID_ARG


def test_argument_errors_before_any_launch(lib):
    # null pointers and bad shapes are rejected on the host, before any CUDA call
    assert lib.llmint8_linear(None, 16, 1024, None, None, 1024, None, None,
                              ctypes.c_float(6.0), 0, None, None, 0, None, None) == \
        llmint8.ERR_INVALID_ARG
    assert lib.llmint8_dequant(None, None, 16, 16, None, None) == llmint8.ERR_INVALID_ARG


def test_empty_and_out_of_range_shapes_are_rejected_before_any_launch(lib):
    fake = ctypes.c_void_p(1 << 20)      # aligned, never dereferenced
    for M, K, N in ((0, 1024, 1024), (16, 0, 1024), (16, 1024, 0), (16, 262144, 1024),
                    (16, 1000, 1024), (16, 1024, 1000)):
        assert lib.llmint8_linear(fake, M, K, fake, fake, N, None, None, ctypes.c_float(6.0),
                                  0, fake, fake, 1 << 20, None, None) == \
            llmint8.ERR_UNSUPPORTED_SHAPE, (M, K, N)
    assert lib.llmint8_quantize_weight_colwise(fake, 0, 1024, fake, fake, None) == \
        llmint8.ERR_UNSUPPORTED_SHAPE
    assert lib.llmint8_dequant(fake, fake, 16, 8, fake, None) == llmint8.ERR_UNSUPPORTED_SHAPE


def test_host_entry_checks_run_before_any_copy(lib):
    # llmint8_linear_host: null host pointers, bad shapes and a short workspace are rejected on
    # the host with llmint8_linear's codes, before the first copy
    fake = ctypes.c_void_p(1 << 20)      # aligned, never dereferenced
    f6 = ctypes.c_float(6.0)
    assert lib.llmint8_linear_host(None, 16, 1024, fake, fake, 1024, None, None, f6, 0, fake,
                                   fake, fake, fake, 1 << 30, None) == llmint8.ERR_INVALID_ARG
    assert lib.llmint8_linear_host(fake, 16, 1024, fake, fake, 1024, None, None, f6, 0, None,
                                   fake, fake, fake, 1 << 30, None) == llmint8.ERR_INVALID_ARG
    assert lib.llmint8_linear_host(fake, 16, 1024, fake, fake, 1024, None, None, f6, 0, fake,
                                   None, fake, fake, 1 << 30, None) == llmint8.ERR_INVALID_ARG
    assert lib.llmint8_linear_host(fake, 16, 1024, fake, fake, 1024, None, None, f6, 0, fake,
                                   ctypes.c_void_p((1 << 20) + 8), fake, fake, 1 << 30,
                                   None) == llmint8.ERR_INVALID_ARG       # X_dev misaligned
    assert lib.llmint8_linear_host(fake, 16, 1000, fake, fake, 1024, None, None, f6, 0, fake,
                                   fake, fake, fake, 1 << 30, None) == \
        llmint8.ERR_UNSUPPORTED_SHAPE
    assert lib.llmint8_linear_host(fake, 16, 1024, fake, fake, 1024, None, None, f6, 0, fake,
                                   fake, fake, fake, 256, None) == \
        llmint8.ERR_WORKSPACE_TOO_SMALL
    assert lib.llmint8_linear_host(fake, 16, 1024, fake, fake, 1024, None, None,
                                   ctypes.c_float(float("nan")), 0, fake, fake, fake, fake,
                                   1 << 30, None) == llmint8.ERR_INVALID_ARG


def test_token_parallel_entries_check_arguments_before_any_launch(lib):
    fake = ctypes.c_void_p(1 << 20)      # aligned, never dereferenced
    f6 = ctypes.c_float(6.0)
    ob = lib.llmint8_outlier_bitmap
    assert ob(None, 16, 1024, f6, fake, fake, 1 << 30, None) == llmint8.ERR_INVALID_ARG
    assert ob(fake, 16, 1024, f6, None, fake, 1 << 30, None) == llmint8.ERR_INVALID_ARG
    assert ob(fake, 16, 1024, ctypes.c_float(float("nan")), fake, fake, 1 << 30, None) == \
        llmint8.ERR_INVALID_ARG
    assert ob(fake, 16, 1000, f6, fake, fake, 1 << 30, None) == llmint8.ERR_UNSUPPORTED_SHAPE
    assert ob(fake, 0, 1024, f6, fake, fake, 1 << 30, None) == llmint8.ERR_UNSUPPORTED_SHAPE
    assert ob(fake, 16, 1024, f6, fake, fake, 64, None) == llmint8.ERR_WORKSPACE_TOO_SMALL
    # the bitmap call's workspace also lists every column: at least 4 K bytes
    assert llmint8.llmint8_quantize_workspace_size(16, 1024) >= 4 * 1024

    wb = lib.llmint8_linear_with_bitmaps

    def call(bitmaps=fake, n=1, K=1024, N=1024, ws_bytes=1 << 30, cap=0):
        return wb(fake, 16, K, fake, fake, N, None, None, bitmaps, n, cap, fake, fake,
                  ws_bytes, None, None)
    assert call(bitmaps=None) == llmint8.ERR_INVALID_ARG
    assert call(bitmaps=ctypes.c_void_p((1 << 20) + 2)) == llmint8.ERR_INVALID_ARG
    assert call(n=0) == llmint8.ERR_INVALID_ARG
    assert call(n=65537) == llmint8.ERR_INVALID_ARG
    assert call(K=1000) == llmint8.ERR_UNSUPPORTED_SHAPE
    assert call(N=1000) == llmint8.ERR_UNSUPPORTED_SHAPE
    assert call(cap=2048) == llmint8.ERR_INVALID_ARG
    assert call(ws_bytes=256) == llmint8.ERR_WORKSPACE_TOO_SMALL
