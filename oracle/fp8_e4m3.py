"""OCP 8-bit floating point, E4M3 variant: a codec written from the format's definition.

TEST INFRASTRUCTURE (see ``oracle/__init__``).

The pages only say that a quantised KV cache stores one byte per value
(page "5.KV Cache 管理 & PagedAttention", Q1, section 1.3 "扩展到量化缓存": FP8
means dtype_bytes = 1).  The encoding itself is the OCP "OFP8" E4M3 format:

* bit 7 sign, bits 6..3 exponent field E (bias 7), bits 2..0 mantissa M;
* E == 0: subnormal, value = (M / 8) * 2**(1 - 7);
* 0 < E: normal, value = (1 + M / 8) * 2**(E - 7);
* E == 15 and M == 7 (S.1111.111) is NaN; there are no infinities, so the
  largest finite magnitude is S.1111.110 = 1.75 * 2**8 = 448.

Encoding used by the cache write: round to nearest, ties to the code whose
mantissa LSB is 0 ("even"), with saturation of finite values beyond +-448 to
+-448 ("satfinite"); NaN maps to 0x7F.  The input is an fp32 number, and the
rounding decision is taken on that fp32 value.
"""

from __future__ import annotations

import math

import numpy as np

EXP_BIAS = 7
MAX_FINITE = 448.0
NAN_CODE = 0x7F


def code_value(code: int) -> float:
    """Value of one E4M3 code, from the bit-field definition above."""
    sign = (code >> 7) & 1
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        mag = (m / 8.0) * 2.0 ** (1 - EXP_BIAS)
    else:
        mag = (1.0 + m / 8.0) * 2.0 ** (e - EXP_BIAS)
    return -mag if sign else mag


# All 256 codes decoded once (fp64 holds every E4M3 value exactly).
VALUES = np.array([code_value(c) for c in range(256)], dtype=np.float64)

# Non-negative finite codes 0x00..0x7E have strictly increasing values.
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALUES = VALUES[:0x7F]


def decode(codes: np.ndarray) -> np.ndarray:
    """uint8 codes -> fp64 values (NaN for the two NaN codes)."""
    return VALUES[np.asarray(codes, dtype=np.uint8).astype(np.int64)]


def encode(x: np.ndarray) -> np.ndarray:
    """fp32 values -> uint8 codes: nearest E4M3 value, ties to even, saturating.

    The nearest value is found by comparing |x| with the exact midpoint of the
    two neighbouring representable magnitudes (midpoints of E4M3 values and
    fp32 inputs are exact in fp64, so the comparison is exact).
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    nan = np.isnan(a)
    a = np.where(nan, 0.0, np.minimum(a, MAX_FINITE))
    # hi = index of the first representable magnitude >= a
    hi = np.searchsorted(_POS_VALUES, a, side="left")
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    v_hi = _POS_VALUES[hi]
    v_lo = _POS_VALUES[lo]
    mid = (v_lo + v_hi) / 2.0
    exact_hi = a == v_hi
    pick_hi = exact_hi | (a > mid) | ((a == mid) & (_POS_CODES[hi] % 2 == 0))
    mag_code = np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo])
    sign = np.signbit(x).astype(np.int64) << 7
    code = np.where(nan, NAN_CODE, mag_code | sign)
    return code.astype(np.uint8)
