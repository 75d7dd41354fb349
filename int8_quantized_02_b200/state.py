"""Saving and loading the int8 state of a layer: CB, SCB, the threshold and the bias.

The blog ("A gentle introduction to 8-bit matrix multiplication...", section 改进范围,
"在 Hub 上保存 8 位状态字典") names as missing that the quantization statistics CB and SCB
are not kept with a saved state, so an 8-bit layer cannot be reloaded directly.  This file
format keeps them.

Layout (little-endian), written and read by this module only:
    0   8 bytes  magic b"LLMINT8W"
    8   u32      format version (1)
    12  u32      flags: bit 0 = a bias follows
    16  i64      N (output channels)
    24  i64      K (input features)
    32  f32      threshold
    36  u32      CRC-32 of everything after the 40-byte header
    40  f32[N]   SCB (absmax per output channel)
        i8[N*K]  CB, row-major (row n = output channel n)
        f16[N]   bias (only with flag bit 0)
"""
from __future__ import annotations

import struct
import zlib

import numpy as np

MAGIC = b"LLMINT8W"
VERSION = 1
_HEADER = struct.Struct("<8sIIqqfI")


class StateFormatError(ValueError):
    """The file is not an int8 layer state of this format, or it is damaged."""


def _host(a, dtype) -> np.ndarray:
    if hasattr(a, "detach"):            # a torch tensor on any device
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=dtype)


def save_int8_weight(path: str, CB, SCB, threshold: float = 6.0, bias=None) -> None:
    """Writes CB int8 [N, K], SCB fp32 [N], the threshold and an optional fp16 bias [N]."""
    CB = _host(CB, np.int8)
    SCB = _host(SCB, np.float32)
    if CB.ndim != 2 or SCB.shape != (CB.shape[0],):
        raise ValueError("CB must be [N, K] and SCB [N]")
    N, K = CB.shape
    parts = [SCB.tobytes(), CB.tobytes()]
    flags = 0
    if bias is not None:
        b = _host(bias, np.float16)
        if b.shape != (N,):
            raise ValueError("bias must be [N]")
        parts.append(b.tobytes())
        flags |= 1
    payload = b"".join(parts)
    header = _HEADER.pack(MAGIC, VERSION, flags, N, K, float(threshold),
                          zlib.crc32(payload) & 0xFFFFFFFF)
    with open(path, "wb") as f:
        f.write(header)
        f.write(payload)


def load_int8_weight(path: str, device=None) -> dict:
    """Reads a state written by save_int8_weight.  Returns numpy arrays, or torch tensors on
    `device` when one is given: {"CB", "SCB", "threshold", "bias" (or None)}."""
    with open(path, "rb") as f:
        data = f.read()
    if len(data) < _HEADER.size:
        raise StateFormatError("file shorter than the header")
    magic, version, flags, N, K, threshold, crc = _HEADER.unpack_from(data, 0)
    if magic != MAGIC:
        raise StateFormatError("not an int8 layer state (bad magic)")
    if version != VERSION:
        raise StateFormatError(f"unsupported format version {version}")
    if N < 1 or K < 1:
        raise StateFormatError("bad shape in header")
    has_bias = bool(flags & 1)
    size = 4 * N + N * K + (2 * N if has_bias else 0)
    payload = data[_HEADER.size:]
    if len(payload) != size:
        raise StateFormatError(f"payload is {len(payload)} bytes, the header implies {size}")
    if zlib.crc32(payload) & 0xFFFFFFFF != crc:
        raise StateFormatError("checksum mismatch")
    SCB = np.frombuffer(payload, np.float32, N, 0).copy()
    CB = np.frombuffer(payload, np.int8, N * K, 4 * N).reshape(N, K).copy()
    bias = np.frombuffer(payload, np.float16, N, 4 * N + N * K).copy() if has_bias else None
    out = {"CB": CB, "SCB": SCB, "threshold": float(threshold), "bias": bias}
    if device is not None:
        import torch
        for k in ("CB", "SCB", "bias"):
            if out[k] is not None:
                out[k] = torch.from_numpy(out[k]).to(device)
    return out
