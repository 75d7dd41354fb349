"""ctypes front end of the CPU oracle (``llmint8_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the benchmark's
CPU-baseline leg are the only callers.  The product path never imports this module.

Every function takes and returns numpy arrays: fp16 tensors as ``np.float16``, int8 as
``np.int8``, scales as ``np.float32``.  The arithmetic lives in the C file; this module
only marshals arguments and builds the shared object with gcc when it is missing or older
than its source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "llmint8_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK = 0
ERR_INVALID_ARG = 1
ERR_OUTLIER_CAPACITY = 4
ERR_INT32_OVERFLOW = 7

# -ffp-contract=off keeps every fp32 multiply a separate rounding step.
CFLAGS = ["-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
          "-fPIC", "-shared"]


def build(src: str = _SRC, out: str = _LIB_PATH, force: bool = False) -> str:
    """Compile the oracle with gcc (no-op when the library is newer than the source)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, src, "-lm"], check=True)
    os.replace(tmp, out)
    return out


def _declare(lib):
    p, i64, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
    lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_half_to_double.restype = ctypes.c_double
    lib.oracle_double_to_half.argtypes = [ctypes.c_double]
    lib.oracle_double_to_half.restype = ctypes.c_uint16
    lib.oracle_quantize_weight_colwise.argtypes = [p, i64, i64, p, p]
    lib.oracle_quantize_rows_and_find_outliers.argtypes = [p, i64, i64, f32, p, p, p, p, i64]
    lib.oracle_int8_accumulate.argtypes = [p, i64, i64, p, i64, p]
    lib.oracle_dequant.argtypes = [p, p, i64, i64, p]
    lib.oracle_linear.argtypes = [p, i64, i64, p, p, i64, p, p, f32, p, p]
    lib.oracle_linear_sampled.argtypes = [p, i64, i64, p, p, i64, p, p, f32, i64, p, p, p, p]
    for name in ("oracle_quantize_weight_colwise", "oracle_quantize_rows_and_find_outliers",
                 "oracle_int8_accumulate", "oracle_dequant", "oracle_linear",
                 "oracle_linear_sampled"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle shared object."""
    global _lib
    with _lock:
        if path is not None:
            return _declare(ctypes.CDLL(path))
        if _lib is None:
            _lib = _declare(ctypes.CDLL(build()))
        return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _f16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.float16, f"expected float16, got {a.dtype}"
    return a


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: oracle status {code}")
        self.code = code


def _check(code: int, what: str, allow=(OK,)):
    if code not in allow:
        raise OracleError(code, what)
    return code


def half_to_double(bits: int, lib=None) -> float:
    return (lib or load()).oracle_half_to_double(bits)


def double_to_half(x: float, lib=None) -> int:
    return (lib or load()).oracle_double_to_half(x)


def quantize_weight_colwise(W: np.ndarray, lib=None):
    """W fp16 [N, K] -> (CB int8 [N, K], SCB fp32 [N] absmax per output row)."""
    lib = lib or load()
    W = _f16(W)
    N, K = W.shape
    CB = np.empty((N, K), np.int8)
    SCB = np.empty((N,), np.float32)
    _check(lib.oracle_quantize_weight_colwise(_ptr(W), N, K, _ptr(CB), _ptr(SCB)),
           "quantize_weight_colwise")
    return CB, SCB


def quantize_rows_and_find_outliers(X: np.ndarray, threshold: float, cap: int | None = None,
                                    lib=None):
    """X fp16 [M, K] -> (Xq int8 [M, K], SCA fp32 [M], outlier columns int32 ascending).

    Raises OracleError(ERR_OUTLIER_CAPACITY) when more than ``cap`` columns qualify.
    """
    lib = lib or load()
    X = _f16(X)
    M, K = X.shape
    cap = K if cap is None else cap
    Xq = np.empty((M, K), np.int8)
    SCA = np.empty((M,), np.float32)
    idx = np.empty((max(cap, 1),), np.int32)
    n = ctypes.c_int32(0)
    _check(lib.oracle_quantize_rows_and_find_outliers(
        _ptr(X), M, K, ctypes.c_float(threshold), _ptr(Xq), _ptr(SCA), _ptr(idx),
        ctypes.byref(n), cap), "quantize_rows_and_find_outliers")
    return Xq, SCA, idx[: n.value].copy()


def int8_accumulate(Xq: np.ndarray, CB: np.ndarray, lib=None) -> np.ndarray:
    """C[i, n] = sum_k Xq[i, k] * CB[n, k] (int32, checked)."""
    lib = lib or load()
    Xq = np.ascontiguousarray(Xq, np.int8)
    CB = np.ascontiguousarray(CB, np.int8)
    M, K = Xq.shape
    N = CB.shape[0]
    C = np.empty((M, N), np.int32)
    _check(lib.oracle_int8_accumulate(_ptr(Xq), M, K, _ptr(CB), N, _ptr(C)), "int8_accumulate")
    return C


def dequant(CB: np.ndarray, SCB: np.ndarray, lib=None) -> np.ndarray:
    """W_hat fp16 [N, K] = fp16((CB * SCB) / 127)."""
    lib = lib or load()
    CB = np.ascontiguousarray(CB, np.int8)
    SCB = np.ascontiguousarray(SCB, np.float32)
    N, K = CB.shape
    out = np.empty((N, K), np.float16)
    _check(lib.oracle_dequant(_ptr(CB), _ptr(SCB), N, K, _ptr(out)), "dequant")
    return out


def linear(X, CB, SCB, bias=None, W_fp16=None, threshold: float = 6.0, want_C: bool = False,
           lib=None):
    """Full layer: Y fp16 [M, N] (and the int32 accumulators C [M, N] when asked)."""
    lib = lib or load()
    X = _f16(X)
    CB = np.ascontiguousarray(CB, np.int8)
    SCB = np.ascontiguousarray(SCB, np.float32)
    bias = None if bias is None else _f16(bias)
    W_fp16 = None if W_fp16 is None else _f16(W_fp16)
    M, K = X.shape
    N = CB.shape[0]
    Y = np.empty((M, N), np.float16)
    C = np.empty((M, N), np.int32) if want_C else None
    _check(lib.oracle_linear(_ptr(X), M, K, _ptr(CB), _ptr(SCB), N, _ptr(bias), _ptr(W_fp16),
                             ctypes.c_float(threshold), _ptr(Y), _ptr(C)), "linear")
    return (Y, C) if want_C else Y


def linear_sampled(X, CB, SCB, rows, cols, bias=None, W_fp16=None, threshold: float = 6.0,
                   lib=None):
    """The layer at the listed output positions only: (Y fp16 [S], C int32 [S])."""
    lib = lib or load()
    X = _f16(X)
    CB = np.ascontiguousarray(CB, np.int8)
    SCB = np.ascontiguousarray(SCB, np.float32)
    bias = None if bias is None else _f16(bias)
    W_fp16 = None if W_fp16 is None else _f16(W_fp16)
    rows = np.ascontiguousarray(rows, np.int64)
    cols = np.ascontiguousarray(cols, np.int64)
    M, K = X.shape
    N = CB.shape[0]
    S = rows.shape[0]
    Y = np.empty((S,), np.float16)
    C = np.empty((S,), np.int32)
    _check(lib.oracle_linear_sampled(_ptr(X), M, K, _ptr(CB), _ptr(SCB), N, _ptr(bias),
                                     _ptr(W_fp16), ctypes.c_float(threshold), S, _ptr(rows),
                                     _ptr(cols), _ptr(Y), _ptr(C)), "linear_sampled")
    return Y, C
