"""INT8 / INT4 KV codes -> float64 values, from two's complement.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The ORT CPU GQA analysis (its introduction and the tiled-loop code block, where V is
dequantised on the fly inside the SV accumulation) names INT8 and INT4 quantised KV
caches but gives no encoding.  Readings taken here, the plainest ones:
  * INT8: one signed two's complement byte per element (-128..127);
  * INT4: two signed 4-bit two's complement elements per byte (-8..7), element 2i of a
    row in the low nibble of byte i and element 2i+1 in the high nibble, so a D-element
    row is D/2 bytes;
  * the element's value is its integer times the float32 scale of its (token, KV head),
    the same per-token scale layout as the FP8 cache.
Attention over the values is then oracle.attention.decode (k_scale / v_scale multiply K and
V rows there).
"""
from __future__ import annotations

import numpy as np


def _u8(codes) -> np.ndarray:
    if hasattr(codes, "detach"):
        codes = codes.detach().cpu()
        if str(codes.dtype) != "torch.uint8":
            codes = codes.view(__import__("torch").uint8)
        codes = codes.numpy()
    return np.asarray(codes).astype(np.uint8, copy=False)


def int8_values(codes) -> np.ndarray:
    """Bytes (uint8 or int8, numpy or torch) -> the two's complement integers as float64."""
    u = _u8(codes).astype(np.int64)
    return np.where(u >= 128, u - 256, u).astype(np.float64)


def int4_values(packed) -> np.ndarray:
    """Packed rows [..., D/2] bytes -> [..., D] float64: low nibble first, each nibble a 4-bit
    two's complement integer."""
    u = _u8(packed).astype(np.int64)
    lo = u & 0xF
    hi = u >> 4
    out = np.empty(u.shape[:-1] + (2 * u.shape[-1],), dtype=np.float64)
    out[..., 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[..., 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out


def int_values(codes, bits: int) -> np.ndarray:
    """Dispatch on the code width (8 or 4)."""
    if bits == 8:
        return int8_values(codes)
    if bits == 4:
        return int4_values(codes)
    raise ValueError(f"unsupported code width {bits}")
