"""E4M3 (OCP FP8, "fn" variant: no infinities) code -> float64, from the format's definition.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The LLM-CoOpt summary ("Opt-KV") stores the KV cache in FP8 and says nothing about
the encoding; the reading taken here is E4M3 with one float32 scale per
(token, KV head).  A code is s eeee mmm: sign s, 4-bit exponent e with bias 7,
3-bit mantissa m.
  e > 0:          (-1)^s * 2^(e-7) * (1 + m/8)
  e = 0:          (-1)^s * 2^(-6) * (m/8)          (subnormals, and +-0)
  e = 15, m = 7:  NaN (the only non-finite codes: 0x7F and 0xFF)
"""
from __future__ import annotations

import numpy as np


def e4m3_value(code: int) -> float:
    code = int(code) & 0xFF
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (2.0 ** -6) * (m / 8.0)
    return s * (2.0 ** (e - 7)) * (1.0 + m / 8.0)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_decode(codes) -> np.ndarray:
    """Decode an array of uint8 codes (numpy or torch) to float64 values."""
    if hasattr(codes, "detach"):
        codes = codes.detach().cpu().numpy()
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]
