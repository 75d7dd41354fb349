"""Python binding of the C ABI in ``include/llmint8.h`` (argument marshalling only).

Every function here takes torch CUDA tensors, allocates any missing output or workspace
with torch, and calls the entry point of the same name in ``libllmint8.so`` on the
current torch stream.  All arithmetic runs in the library's sm_100a kernels; there is no
fallback: a missing library raises ``LLMInt8LibraryError``.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

# LLMINT8_DEBUG=1 selects the debug build (device-side bounds checks; see llmint8_build_flags)
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         "libllmint8_debug.so" if os.environ.get("LLMINT8_DEBUG") == "1"
                         else "libllmint8.so")
_lock = threading.Lock()
_lib = None

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED_SHAPE = 2
ERR_WORKSPACE_TOO_SMALL = 3
ERR_OUTLIER_CAPACITY = 4
ERR_TIMEOUT = 5
ERR_CUDA = 6
ERR_DEVICE_CHECK = 7

# Names and prototypes exactly as declared in include/llmint8.h.
_P, _I64, _F32, _SZ, _U64 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t,
                             ctypes.c_uint64)
PROTOTYPES = {
    "llmint8_quantize_weight_colwise": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P]),
    "llmint8_quantize_rows_and_find_outliers": (
        ctypes.c_int, [_P, _I64, _I64, _F32, _P, _P, _P, _P, _I64, _P, _SZ, _P]),
    "llmint8_quantize_workspace_size": (_SZ, [_I64, _I64]),
    "llmint8_linear": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _I64, _P, _P, _F32, _I64, _P, _P,
                                      _SZ, _P, _P]),
    "llmint8_linear_next_bitmaps": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _I64, _P, _P, _F32,
                                                   _I64, _P, _P, _SZ, _P, _P, _F32, _P]),
    "llmint8_linear_workspace_size": (_SZ, [_I64, _I64, _I64, _I64]),
    "llmint8_dequant": (ctypes.c_int, [_P, _P, _I64, _I64, _P, _P]),
    "llmint8_device_status": (ctypes.c_int, [_P, _P]),
    "llmint8_workspace_outlier_count": (ctypes.c_int, [_P, _P, _P]),
    "llmint8_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "llmint8_build_flags": (ctypes.c_int, []),
    "llmint8_set_wait_timeout_ns": (ctypes.c_int, [_U64]),
    "llmint8_set_profile_events": (ctypes.c_int, [_P, _P]),
    "llmint8_kernel_launch_count": (_U64, []),
    "llmint8_linear_noalloc": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _I64, _P, _P, _F32, _I64,
                                              _P, _P, ctypes.POINTER(ctypes.c_void_p)]),
    "llmint8_linear_host": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _I64, _P, _P, _F32, _I64, _P,
                                           _P, _P, _P, _SZ, _P]),
    "llmint8_outlier_bitmap": (ctypes.c_int, [_P, _I64, _I64, _F32, _P, _P, _SZ, _P]),
    "llmint8_workspace_outlier_weights": (ctypes.c_int, [_P, _I64, _I64, _I64, _I64, _P, _I64,
                                                         _P]),
    "llmint8_linear_with_bitmaps": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _I64, _P, _P, _P, _I64,
                                                   _I64, _P, _P, _SZ, _P, _P]),
}


class LLMInt8LibraryError(RuntimeError):
    """The compiled library is missing or does not load."""


class LLMInt8Error(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} (status {code})")
        self.code = code


def library_path() -> str:
    return _LIB_PATH


def load():
    """The ctypes handle of libllmint8.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise LLMInt8LibraryError(
                    f"{_LIB_PATH} is missing; build it with `python -m int8_quantized_02_b200.build`")
            try:
                lib = ctypes.CDLL(_LIB_PATH)
            except OSError as e:  # pragma: no cover - depends on the machine
                raise LLMInt8LibraryError(str(e)) from e
            for name, (res, args) in PROTOTYPES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
        return _lib


def status_string(code: int) -> str:
    return load().llmint8_status_string(int(code)).decode()


def build_flags() -> int:
    """llmint8_build_flags(): bit 0 set when the loaded library is the debug build."""
    return int(load().llmint8_build_flags())


llmint8_status_string = status_string


def _check(code: int, what: str):
    if code != OK:
        raise LLMInt8Error(code, what)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("llmint8 tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("llmint8 tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _host_ptr(t: torch.Tensor):
    if t.is_cuda:
        raise ValueError("host buffers must be CPU tensors")
    if not t.is_contiguous():
        raise ValueError("llmint8 tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _want(t: torch.Tensor, dtype: torch.dtype, shape, name: str):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def default_max_outliers(K: int, threshold: float) -> int:
    """Capacity used when the caller gives none: every column when the threshold marks
    all of them (threshold <= 0), else min(K, 512)."""
    return K if threshold <= 0 else min(K, 512)


def llmint8_quantize_workspace_size(M: int, K: int) -> int:
    return int(load().llmint8_quantize_workspace_size(M, K))


def llmint8_linear_workspace_size(M: int, N: int, K: int, max_outliers: int) -> int:
    return int(load().llmint8_linear_workspace_size(M, N, K, max_outliers))


def llmint8_quantize_weight_colwise(W: torch.Tensor, CB=None, SCB=None, stream=None):
    """W fp16 [N, K] -> (CB int8 [N, K], SCB fp32 [N])."""
    N, K = W.shape
    _want(W, torch.float16, (N, K), "W")
    CB = torch.empty((N, K), dtype=torch.int8, device=W.device) if CB is None else CB
    SCB = torch.empty((N,), dtype=torch.float32, device=W.device) if SCB is None else SCB
    _want(CB, torch.int8, (N, K), "CB")
    _want(SCB, torch.float32, (N,), "SCB")
    _check(load().llmint8_quantize_weight_colwise(_ptr(W), N, K, _ptr(CB), _ptr(SCB),
                                                  _stream(stream)),
           "llmint8_quantize_weight_colwise")
    return CB, SCB


def llmint8_quantize_rows_and_find_outliers(X: torch.Tensor, threshold: float = 6.0,
                                            cap: int | None = None, workspace=None,
                                            stream=None):
    """X fp16 [M, K] -> (Xq int8 [M, K], SCA fp32 [M], outlier_idx int32 [cap],
    n_outliers int32 [1], workspace).  The first n_outliers entries of outlier_idx are valid."""
    M, K = X.shape
    _want(X, torch.float16, (M, K), "X")
    cap = K if cap is None else int(cap)
    dev = X.device
    Xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    SCA = torch.empty((M,), dtype=torch.float32, device=dev)
    idx = torch.empty((max(cap, 1),), dtype=torch.int32, device=dev)
    cnt = torch.empty((1,), dtype=torch.int32, device=dev)
    need = llmint8_quantize_workspace_size(M, K)
    ws = torch.empty((need,), dtype=torch.uint8, device=dev) if workspace is None else workspace
    _check(load().llmint8_quantize_rows_and_find_outliers(
        _ptr(X), M, K, ctypes.c_float(threshold), _ptr(Xq), _ptr(SCA), _ptr(idx), _ptr(cnt), cap,
        _ptr(ws), ws.numel(), _stream(stream)), "llmint8_quantize_rows_and_find_outliers")
    return Xq, SCA, idx, cnt, ws


def llmint8_linear(X: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor, bias=None, W_fp16=None,
                   threshold: float = 6.0, max_outliers: int | None = None, Y=None,
                   workspace=None, C_debug=None, stream=None):
    """The LLM.int8() layer: Y fp16 [M, N] from X fp16 [M, K] and the int8 weight (CB, SCB)."""
    M, K = X.shape
    N = CB.shape[0]
    _want(X, torch.float16, (M, K), "X")
    _want(CB, torch.int8, (N, K), "CB")
    _want(SCB, torch.float32, (N,), "SCB")
    if bias is not None:
        _want(bias, torch.float16, (N,), "bias")
    if W_fp16 is not None:
        _want(W_fp16, torch.float16, (N, K), "W_fp16")
    if C_debug is not None:
        _want(C_debug, torch.int32, (M, N), "C_debug")
    cap = default_max_outliers(K, threshold) if max_outliers is None else int(max_outliers)
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if Y is None else Y
    _want(Y, torch.float16, (M, N), "Y")
    if workspace is None:
        workspace = torch.empty((llmint8_linear_workspace_size(M, N, K, cap),), dtype=torch.uint8,
                                device=X.device)
    _check(load().llmint8_linear(_ptr(X), M, K, _ptr(CB), _ptr(SCB), N, _ptr(bias), _ptr(W_fp16),
                                 ctypes.c_float(threshold), cap, _ptr(Y), _ptr(workspace),
                                 workspace.numel(), _stream(stream), _ptr(C_debug)),
           "llmint8_linear")
    return Y


def llmint8_linear_next_bitmaps(X: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor,
                                next_threshold: float = 6.0, bias=None, W_fp16=None,
                                threshold: float = 6.0, max_outliers: int | None = None, Y=None,
                                next_bitmaps=None, workspace=None, C_debug=None, stream=None):
    """llmint8_linear that also returns the outlier bitmaps of Y for a next layer taking Y as
    its input: (Y, bitmaps uint32 [ceil(M/32), ceil(N/32)]), ready for that layer's
    llmint8_linear_with_bitmaps."""
    M, K = X.shape
    N = CB.shape[0]
    _want(X, torch.float16, (M, K), "X")
    _want(CB, torch.int8, (N, K), "CB")
    _want(SCB, torch.float32, (N,), "SCB")
    if bias is not None:
        _want(bias, torch.float16, (N,), "bias")
    if W_fp16 is not None:
        _want(W_fp16, torch.float16, (N, K), "W_fp16")
    if C_debug is not None:
        _want(C_debug, torch.int32, (M, N), "C_debug")
    cap = default_max_outliers(K, threshold) if max_outliers is None else int(max_outliers)
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if Y is None else Y
    _want(Y, torch.float16, (M, N), "Y")
    shape = ((M + 31) // 32, (N + 31) // 32)
    if next_bitmaps is None:
        next_bitmaps = torch.empty(shape, dtype=torch.int32, device=X.device)
    if next_bitmaps.dtype not in (torch.int32, torch.uint32) or \
            tuple(next_bitmaps.shape) != shape or not next_bitmaps.is_contiguous():
        raise ValueError(f"next_bitmaps: want a contiguous 32-bit tensor of shape {shape}")
    if workspace is None:
        workspace = torch.empty((llmint8_linear_workspace_size(M, N, K, cap),), dtype=torch.uint8,
                                device=X.device)
    _check(load().llmint8_linear_next_bitmaps(
        _ptr(X), M, K, _ptr(CB), _ptr(SCB), N, _ptr(bias), _ptr(W_fp16), ctypes.c_float(threshold),
        cap, _ptr(Y), _ptr(workspace), workspace.numel(), _stream(stream), _ptr(C_debug),
        ctypes.c_float(next_threshold), _ptr(next_bitmaps)), "llmint8_linear_next_bitmaps")
    return Y, next_bitmaps


def llmint8_linear_fp16_weight(X: torch.Tensor, W: torch.Tensor, bias=None,
                               threshold: float = 6.0, max_outliers: int | None = None, Y=None,
                               workspace=None, CB=None, SCB=None, stream=None):
    """The layer with fp16 weights kept (the blog's has_fp16_weights=True, section 用法):
    every call quantizes W per output channel (CB, SCB) and the outlier columns use the
    original fp16 rows of W.  Two calls of the C ABI, both on the GPU:
    llmint8_quantize_weight_colwise, then llmint8_linear with W_fp16 = W."""
    CB, SCB = llmint8_quantize_weight_colwise(W, CB, SCB, stream)
    return llmint8_linear(X, CB, SCB, bias=bias, W_fp16=W, threshold=threshold,
                          max_outliers=max_outliers, Y=Y, workspace=workspace, stream=stream)


class LinearPlan:
    """One llmint8_linear call with its arguments checked and marshalled once.

    Calling the plan launches the same C entry point with the same tensors, so a loop that
    runs the layer on fixed buffers (a decode loop) pays the Python-side argument handling
    only once.  The tensors must stay alive and keep their storage while the plan is used."""

    def __init__(self, X: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor, bias=None,
                 W_fp16=None, threshold: float = 6.0, max_outliers: int | None = None, Y=None,
                 workspace=None, C_debug=None, stream=None):
        M, K = X.shape
        N = CB.shape[0]
        _want(X, torch.float16, (M, K), "X")
        _want(CB, torch.int8, (N, K), "CB")
        _want(SCB, torch.float32, (N,), "SCB")
        if bias is not None:
            _want(bias, torch.float16, (N,), "bias")
        if W_fp16 is not None:
            _want(W_fp16, torch.float16, (N, K), "W_fp16")
        if C_debug is not None:
            _want(C_debug, torch.int32, (M, N), "C_debug")
        cap = default_max_outliers(K, threshold) if max_outliers is None else int(max_outliers)
        self.Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if Y is None else Y
        _want(self.Y, torch.float16, (M, N), "Y")
        if workspace is None:
            workspace = torch.empty((llmint8_linear_workspace_size(M, N, K, cap),),
                                    dtype=torch.uint8, device=X.device)
        self.workspace = workspace
        self._keep = (X, CB, SCB, bias, W_fp16, C_debug)
        self._fn = load().llmint8_linear
        self._args = (_ptr(X), M, K, _ptr(CB), _ptr(SCB), N, _ptr(bias), _ptr(W_fp16),
                      ctypes.c_float(threshold), cap, _ptr(self.Y), _ptr(workspace),
                      workspace.numel(), _stream(stream), _ptr(C_debug))

    def __call__(self) -> torch.Tensor:
        code = self._fn(*self._args)
        if code != OK:
            raise LLMInt8Error(code, "llmint8_linear")
        return self.Y


def bitmap_words(K: int) -> int:
    """uint32 words of an outlier-column bitmap over K columns."""
    return (K + 31) // 32


def llmint8_outlier_bitmap(X: torch.Tensor, threshold: float = 6.0, bitmap=None,
                           workspace=None, stream=None) -> torch.Tensor:
    """X fp16 [M, K] -> int32 [ceil(K/32)] bitmap of its outlier columns (bit j % 32 of word
    j // 32; the words are uint32 bit patterns held in an int32 tensor)."""
    M, K = X.shape
    _want(X, torch.float16, (M, K), "X")
    W = bitmap_words(K)
    bitmap = torch.empty((W,), dtype=torch.int32, device=X.device) if bitmap is None else bitmap
    _want(bitmap, torch.int32, (W,), "bitmap")
    need = llmint8_quantize_workspace_size(M, K)
    ws = torch.empty((need,), dtype=torch.uint8, device=X.device) if workspace is None \
        else workspace
    _check(load().llmint8_outlier_bitmap(_ptr(X), M, K, ctypes.c_float(threshold), _ptr(bitmap),
                                         _ptr(ws), ws.numel(), _stream(stream)),
           "llmint8_outlier_bitmap")
    return bitmap


def llmint8_linear_with_bitmaps(X: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor,
                                bitmaps: torch.Tensor, bias=None, W_fp16=None,
                                max_outliers: int | None = None, Y=None, workspace=None,
                                C_debug=None, stream=None) -> torch.Tensor:
    """The layer with the outlier set given as the OR of `bitmaps` int32 [n, ceil(K/32)]
    (one row per rank of a token-parallel layer)."""
    M, K = X.shape
    N = CB.shape[0]
    _want(X, torch.float16, (M, K), "X")
    _want(CB, torch.int8, (N, K), "CB")
    _want(SCB, torch.float32, (N,), "SCB")
    if bitmaps.dim() == 1:
        bitmaps = bitmaps.view(1, -1)
    _want(bitmaps, torch.int32, (bitmaps.shape[0], bitmap_words(K)), "bitmaps")
    if bias is not None:
        _want(bias, torch.float16, (N,), "bias")
    if W_fp16 is not None:
        _want(W_fp16, torch.float16, (N, K), "W_fp16")
    if C_debug is not None:
        _want(C_debug, torch.int32, (M, N), "C_debug")
    cap = min(K, 512) if max_outliers is None else int(max_outliers)
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if Y is None else Y
    _want(Y, torch.float16, (M, N), "Y")
    if workspace is None:
        workspace = torch.empty((llmint8_linear_workspace_size(M, N, K, cap),), dtype=torch.uint8,
                                device=X.device)
    _check(load().llmint8_linear_with_bitmaps(
        _ptr(X), M, K, _ptr(CB), _ptr(SCB), N, _ptr(bias), _ptr(W_fp16), _ptr(bitmaps),
        bitmaps.shape[0], cap, _ptr(Y), _ptr(workspace), workspace.numel(), _stream(stream),
        _ptr(C_debug)), "llmint8_linear_with_bitmaps")
    return Y


class LinearHostPlan:
    """llmint8_linear_host on fixed buffers: host X in, host Y out, marshalled once.

    Each call copies X_host to the device, runs the layer and copies Y back into Y_host, all
    on the stream; Y_host holds the result once the stream has been synchronized.  Pinned
    host tensors (``pin_memory()``) keep the call asynchronous.  The device staging buffers
    and the workspace are allocated here unless given."""

    def __init__(self, X_host: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor,
                 Y_host: torch.Tensor | None = None, bias=None, W_fp16=None,
                 threshold: float = 6.0, max_outliers: int | None = None, X_dev=None,
                 Y_dev=None, workspace=None, stream=None):
        M, K = X_host.shape
        N = CB.shape[0]
        dev = CB.device
        _want(X_host, torch.float16, (M, K), "X_host")
        _want(CB, torch.int8, (N, K), "CB")
        _want(SCB, torch.float32, (N,), "SCB")
        if bias is not None:
            _want(bias, torch.float16, (N,), "bias")
        if W_fp16 is not None:
            _want(W_fp16, torch.float16, (N, K), "W_fp16")
        cap = default_max_outliers(K, threshold) if max_outliers is None else int(max_outliers)
        self.Y_host = torch.empty((M, N), dtype=torch.float16).pin_memory() \
            if Y_host is None else Y_host
        _want(self.Y_host, torch.float16, (M, N), "Y_host")
        self.X_dev = torch.empty((M, K), dtype=torch.float16, device=dev) if X_dev is None \
            else X_dev
        self.Y_dev = torch.empty((M, N), dtype=torch.float16, device=dev) if Y_dev is None \
            else Y_dev
        _want(self.X_dev, torch.float16, (M, K), "X_dev")
        _want(self.Y_dev, torch.float16, (M, N), "Y_dev")
        if workspace is None:
            workspace = torch.empty((llmint8_linear_workspace_size(M, N, K, cap),),
                                    dtype=torch.uint8, device=dev)
        self.workspace = workspace
        self._keep = (X_host, CB, SCB, bias, W_fp16)
        self._fn = load().llmint8_linear_host
        self._args = (_host_ptr(X_host), M, K, _ptr(CB), _ptr(SCB), N, _ptr(bias),
                      _ptr(W_fp16), ctypes.c_float(threshold), cap, _host_ptr(self.Y_host),
                      _ptr(self.X_dev), _ptr(self.Y_dev), _ptr(workspace), workspace.numel(),
                      _stream(stream))

    def __call__(self) -> torch.Tensor:
        code = self._fn(*self._args)
        if code != OK:
            raise LLMInt8Error(code, "llmint8_linear_host")
        return self.Y_host


def llmint8_linear_host(X_host: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor,
                        Y_host=None, bias=None, W_fp16=None, threshold: float = 6.0,
                        max_outliers: int | None = None, X_dev=None, Y_dev=None, workspace=None,
                        stream=None, synchronize: bool = True) -> torch.Tensor:
    """The layer on a host X fp16 [M, K]: Y fp16 [M, N] in host memory (by default the stream
    is synchronized before returning, so Y is ready)."""
    plan = LinearHostPlan(X_host, CB, SCB, Y_host, bias, W_fp16, threshold, max_outliers,
                          X_dev, Y_dev, workspace, stream)
    Y = plan()
    if synchronize:
        (torch.cuda.current_stream() if stream is None else stream).synchronize()
    return Y


def llmint8_dequant(CB: torch.Tensor, SCB: torch.Tensor, out=None, stream=None):
    """(CB int8 [N, K], SCB fp32 [N]) -> fp16 [N, K] = (CB * SCB) / 127."""
    N, K = CB.shape
    _want(CB, torch.int8, (N, K), "CB")
    _want(SCB, torch.float32, (N,), "SCB")
    out = torch.empty((N, K), dtype=torch.float16, device=CB.device) if out is None else out
    _want(out, torch.float16, (N, K), "out")
    _check(load().llmint8_dequant(_ptr(CB), _ptr(SCB), N, K, _ptr(out), _stream(stream)),
           "llmint8_dequant")
    return out


def llmint8_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronizes the stream; the device status code of the last call on `workspace`."""
    return int(load().llmint8_device_status(_ptr(workspace), _stream(stream)))


def llmint8_workspace_outlier_count(workspace: torch.Tensor, stream=None) -> int:
    n = ctypes.c_int32(0)
    _check(load().llmint8_workspace_outlier_count(_ptr(workspace), _stream(stream),
                                                  ctypes.byref(n)),
           "llmint8_workspace_outlier_count")
    return int(n.value)


def llmint8_workspace_outlier_weights(workspace: torch.Tensor, M: int, N: int, K: int,
                                      max_outliers: int, n_cols: int, stream=None):
    """fp16 [N, n_cols]: the outlier-weight rows the last llmint8_linear call on `workspace`
    (with these M, N, K, max_outliers) used; on the decode path only after a call with
    C_debug."""
    Wo = torch.empty((N, max(int(n_cols), 1)), dtype=torch.float16, device=workspace.device)
    _check(load().llmint8_workspace_outlier_weights(_ptr(workspace), M, N, K, max_outliers,
                                                    _ptr(Wo), int(n_cols), _stream(stream)),
           "llmint8_workspace_outlier_weights")
    return Wo[:, :int(n_cols)]


def llmint8_set_wait_timeout_ns(ns: int) -> None:
    _check(load().llmint8_set_wait_timeout_ns(int(ns)), "llmint8_set_wait_timeout_ns")


def llmint8_set_profile_events(start=None, stop=None) -> None:
    """Record torch.cuda.Event pair (start, stop) around the product kernel of every later
    llmint8_linear call; (None, None) disables."""
    s = None if start is None else ctypes.c_void_p(start.cuda_event)
    e = None if stop is None else ctypes.c_void_p(stop.cuda_event)
    if (start is not None and not start.cuda_event) or (stop is not None and not stop.cuda_event):
        raise ValueError("record the events once before handing them to the library")
    _check(load().llmint8_set_profile_events(s, e), "llmint8_set_profile_events")


def llmint8_kernel_launch_count() -> int:
    return int(load().llmint8_kernel_launch_count())


def llmint8_linear_noalloc(X: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor, Y: torch.Tensor,
                           bias=None, W_fp16=None, threshold: float = 6.0,
                           max_outliers: int = 64, stream=None) -> int:
    """llmint8_linear on the library's fixed per-device scratch: no workspace, nothing
    allocated (the caller passes Y).  Decode shapes only (M <= 16, K <= 16384, threshold > 0,
    max_outliers <= 256).  Returns the device address of the scratch, whose header
    llmint8_device_status / llmint8_workspace_outlier_count read through the C ABI."""
    M, K = X.shape
    N = CB.shape[0]
    _want(X, torch.float16, (M, K), "X")
    _want(CB, torch.int8, (N, K), "CB")
    _want(SCB, torch.float32, (N,), "SCB")
    _want(Y, torch.float16, (M, N), "Y")
    if bias is not None:
        _want(bias, torch.float16, (N,), "bias")
    if W_fp16 is not None:
        _want(W_fp16, torch.float16, (N, K), "W_fp16")
    scratch = ctypes.c_void_p(0)
    _check(load().llmint8_linear_noalloc(_ptr(X), M, K, _ptr(CB), _ptr(SCB), N, _ptr(bias),
                                         _ptr(W_fp16), ctypes.c_float(threshold),
                                         int(max_outliers), _ptr(Y), _stream(stream),
                                         ctypes.byref(scratch)),
           "llmint8_linear_noalloc")
    return int(scratch.value or 0)
