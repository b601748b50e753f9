"""Stored element formats -> exact fp64 values.

TEST INFRASTRUCTURE (see ``oracle/__init__``).

Caches and queries are handed to the oracle as raw storage:

* ``"f16"``  -- IEEE binary16, as ``numpy.float16`` (or its uint16 bits);
* ``"bf16"`` -- bfloat16 bits as ``uint16``: by definition the upper 16 bits of
  an IEEE binary32, so the value is those bits shifted into the top half of a
  32-bit word;
* ``"fp8_e4m3"`` -- OCP E4M3 codes as ``uint8`` (``oracle.fp8_e4m3``).

Every conversion here is exact (each format embeds in fp64).
"""

from __future__ import annotations

import numpy as np

from . import fp8_e4m3

F16, BF16, FP8 = "f16", "bf16", "fp8_e4m3"
ELEMENT_BYTES = {F16: 2, BF16: 2, FP8: 1}


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> fp64."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def to_f64(raw: np.ndarray, dtype: str) -> np.ndarray:
    """Raw storage of the given format -> fp64 array of the same shape."""
    if dtype == F16:
        if raw.dtype == np.float16:
            return raw.astype(np.float64)
        return np.asarray(raw).astype(np.uint16).view(np.float16).astype(np.float64)
    if dtype == BF16:
        return bf16_bits_to_f64(raw)
    if dtype == FP8:
        return fp8_e4m3.decode(raw)
    raise ValueError(f"unknown storage format {dtype!r}")


def to_f32(raw: np.ndarray, dtype: str) -> np.ndarray:
    """16-bit storage -> fp32 (exact: both 16-bit formats embed in binary32)."""
    if dtype not in (F16, BF16):
        raise ValueError("only 16-bit formats convert to fp32 here")
    return to_f64(raw, dtype).astype(np.float32)
