"""E5M2 encoder and decoder, written out from the format.

Format ['FP8量化在生成式推荐系统OneRec-V2中的优化实践' §2.2 names E5M2, 5 exponent
bits and 2 mantissa bits, for the activations]: 1 sign bit, 5 exponent bits
with bias 15, 2 mantissa bits, IEEE-style specials: exponent field 31 with
mantissa 0 is ±infinity, with mantissa 1..3 NaN.  The largest finite
magnitude is 1.75 * 2^15 = 57344 (code 0x7B); exponent field 0 holds
subnormals (m/4) * 2^-14, the smallest being 2^-16.

Encoding reading (the pages fix no rounding mode; the same reading as the
E4M3 codec): round to nearest, ties to even, saturating finite values at or
above 57344 to ±57344 (never to infinity).  -0.0 keeps its sign (0x80).  NaN
maps to 0x7F with the sign bit kept; non-finite inputs are outside the
path's contract.

All arithmetic is float64 on float32 inputs, exact here for the same reason
as in the E4M3 codec; the only rounding is the explicit np.rint (half to
even).
"""
from __future__ import annotations

import numpy as np

E5M2_MAX = 57344.0
_MIN_NORMAL = 2.0 ** -14
_SUB_STEP = 2.0 ** -16
_MAX_CODE = 0x7B


def e5m2_decode(codes) -> np.ndarray:
    """uint8 codes -> float64 values (±inf for 0x7C / 0xFC, NaN for 0x7D-0x7F and 0xFD-0xFF)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 2) & 0x1F
    m = (c & 0x3).astype(np.float64)
    sub = m * _SUB_STEP
    nrm = (1.0 + m / 4.0) * np.ldexp(1.0, (e - 15).astype(np.int64))
    v = sign * np.where(e == 0, sub, nrm)
    v = np.where((e == 31) & (m == 0), sign * np.inf, v)
    return np.where((e == 31) & (m != 0), np.nan, v)


def e5m2_encode(values) -> np.ndarray:
    """float32 values -> uint8 E5M2 codes (RNE, saturating at ±57344)."""
    v32 = np.asarray(values, dtype=np.float32)
    neg = np.signbit(v32)
    t = np.abs(v32.astype(np.float64))
    out = np.zeros(t.shape, dtype=np.int64)

    nan = np.isnan(t)
    sat = (~nan) & (t >= E5M2_MAX)
    sub = (~nan) & (t < _MIN_NORMAL)
    nrm = ~(nan | sat | sub)

    # Subnormals: value = m * 2^-16, m = rne(t / 2^-16) in [0, 4]; m == 4 is
    # the smallest normal, whose code is also 4 (exponent field 1, mantissa 0).
    out[sub] = np.rint(t[sub] / _SUB_STEP).astype(np.int64)

    # Normals: t = f * 2^ex with f in [0.5, 1), unbiased exponent e = ex - 1,
    # t / 2^e in [1, 2); two mantissa bits.
    tn = t[nrm]
    _, ex = np.frexp(tn)
    e = ex.astype(np.int64) - 1
    frac = np.rint((np.ldexp(tn, -e) - 1.0) * 4.0).astype(np.int64)
    carry = frac == 4                     # rounded up into the next binade
    e = e + carry
    frac = np.where(carry, 0, frac)
    code = ((e + 15) << 2) | frac
    out[nrm] = np.minimum(code, _MAX_CODE)

    out[sat] = _MAX_CODE
    out[nan] = 0x7F
    out = out | (neg.astype(np.int64) << 7)
    return out.astype(np.uint8)
