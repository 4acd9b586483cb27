"""Number formats used by the oracle, written from their definitions.

E2M1 (4-bit float: 1 sign, 2 exponent bits, bias 1, 1 mantissa bit) and
E4M3 (8-bit float, OCP "E4M3FN": 1 sign, 4 exponent bits, bias 7, 3 mantissa
bits, no infinities, only S.1111.111 is NaN, max 448) are the element and
block-scale types of NVFP4.  The pages call NVFP4 a 4-bit float with a
"2-bit exponent + 2-bit mantissa" (4-bit quantisation page, section 3.2); that
adds up to 5 bits with the sign, so the oracle takes the standard E2M1 reading.

Encoders are brute force over the code table: every representable value is
listed, the input is rounded to the nearest one, a tie goes to the code whose
mantissa LSB is 0 (round-to-nearest-even), and magnitudes beyond the largest
finite value saturate to it ("satfinite").  The sign bit follows the input's
sign, so a negative value that rounds to zero keeps the sign bit (IEEE -0).
"""
from __future__ import annotations

import numpy as np


def _decode_minifloat(code: int, ebits: int, mbits: int, bias: int) -> float:
    sign = -1.0 if (code >> (ebits + mbits)) & 1 else 1.0
    e = (code >> mbits) & ((1 << ebits) - 1)
    m = code & ((1 << mbits) - 1)
    if e == 0:                                   # subnormal
        return sign * (m / (1 << mbits)) * 2.0 ** (1 - bias)
    return sign * (1.0 + m / (1 << mbits)) * 2.0 ** (e - bias)


# code -> value tables (NaN code of E4M3 marked as nan)
E2M1_VALUES = np.array([_decode_minifloat(c, 2, 1, 1) for c in range(16)], dtype=np.float64)
E4M3_VALUES = np.array([_decode_minifloat(c, 4, 3, 7) for c in range(256)], dtype=np.float64)
E4M3_VALUES[0x7F] = np.nan
E4M3_VALUES[0xFF] = np.nan

E2M1_MAX = 6.0
E4M3_MAX = 448.0


def _encoder(values: np.ndarray, sign_bit: int, max_code: int):
    """Build an RNE-satfinite encoder over the non-negative codes 0..max_code."""
    mags = values[: max_code + 1]
    assert np.all(np.diff(mags) > 0)
    mids = 0.5 * (mags[:-1] + mags[1:])          # decision points between neighbours

    def encode(x: np.ndarray) -> np.ndarray:
        x = np.asarray(x, dtype=np.float64)
        if np.any(~np.isfinite(x)):
            raise ValueError("non-finite input")
        a = np.abs(x)
        # j = number of decision points strictly below a, so
        # mids[j-1] < a <= mids[j]: code j is the nearest unless a == mids[j]
        j = np.searchsorted(mids, a, side="left")
        is_tie = (j < len(mids)) & (a == mids[np.minimum(j, len(mids) - 1)])
        even = np.where(j % 2 == 0, j, j + 1)     # of codes j, j+1 the one with mantissa LSB 0
        code = np.where(is_tie, even, j)
        code = np.minimum(code, max_code)         # satfinite: beyond the top -> largest finite
        return (code | np.where(np.signbit(x), sign_bit, 0)).astype(np.uint8)

    return encode


e2m1_encode = _encoder(E2M1_VALUES, 0x8, 7)
e4m3_encode = _encoder(E4M3_VALUES, 0x80, 0x7E)


def e2m1_decode(code: np.ndarray) -> np.ndarray:
    return E2M1_VALUES[np.asarray(code, dtype=np.int64) & 0xF]


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    return E4M3_VALUES[np.asarray(code, dtype=np.int64) & 0xFF]


def round_to_precision(x: np.ndarray, sig_bits: int, emin: int) -> np.ndarray:
    """Round float64 values to a binary float with `sig_bits` significant bits
    and minimum normal exponent `emin` (values below are rounded on the
    subnormal grid 2^(emin - sig_bits + 1)), round-to-nearest-even, one step.
    No overflow handling: callers stay in range."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                           # |x| = m 2^e, m in [0.5, 1)
    e = np.maximum(e - 1, emin)                  # unbiased exponent of the leading bit
    quantum = np.ldexp(1.0, e - (sig_bits - 1))
    return np.rint(x / quantum) * quantum        # x / quantum is exact (power of two)


def to_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> nearest bf16 value (8 significant bits, emin -126), as float64."""
    y = round_to_precision(x, 8, -126)
    if np.any(np.abs(y) > 3.3895313892515355e38):
        raise OverflowError("bf16 overflow")
    return y


def to_fp16(x: np.ndarray) -> np.ndarray:
    """float64 -> nearest fp16 value (11 significant bits, emin -14), as float64."""
    y = round_to_precision(x, 11, -14)
    if np.any(np.abs(y) > 65504.0):
        raise OverflowError("fp16 overflow")
    return y


def to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    return to_bf16(x) if dtype == "bf16" else to_fp16(x)


def bf16_bits(v: np.ndarray) -> np.ndarray:
    """Bit patterns (uint16) of values that are exactly bf16."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_from_bits(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
