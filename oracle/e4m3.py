"""E4M3 ("fn" variant) encoder and decoder, written out from the format.

Format [P2 §2.2 names E4M3 for the FP8 path; §1.2 gives its range ±448]:
1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; no infinities; the
all-ones pattern S.1111.111 is NaN, so the largest finite magnitude is
1.75 * 2^8 = 448 (code 0x7E).  Exponent field 0 holds subnormals
(m/8) * 2^-6; the smallest subnormal is 2^-9.

Encoding reading (the pages do not fix a rounding mode): round to nearest,
ties to even, saturating finite values above 448 to ±448.  -0.0 keeps its sign
(code 0x80).  NaN maps to 0x7F with the sign bit kept; non-finite inputs are
outside the path's contract.

All arithmetic is float64 on float32 inputs, which is exact here: a float32
has 24 significant bits, so t / 2^e and (t / 2^e - 1) * 8 are exact in
float64 and the only rounding is the explicit np.rint (round half to even).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
_SUBNORMAL_LIMIT = 2.0 ** -6      # smallest normal
_SUBNORMAL_STEP = 2.0 ** -9       # spacing of subnormals
_MAX_CODE = 0x7E


def e4m3_decode(codes) -> np.ndarray:
    """uint8 codes -> float64 values (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    sub = (m / 8.0) * 2.0 ** -6
    # exponent field e >= 1: (1 + m/8) * 2^(e - 7)
    nrm = (1.0 + m / 8.0) * np.ldexp(1.0, (e - 7).astype(np.int64))
    v = sign * np.where(e == 0, sub, nrm)
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


def e4m3_encode(values) -> np.ndarray:
    """float32 values -> uint8 E4M3 codes (RNE, saturating at ±448)."""
    v32 = np.asarray(values, dtype=np.float32)
    neg = np.signbit(v32)
    t = np.abs(v32.astype(np.float64))
    out = np.zeros(t.shape, dtype=np.int64)

    nan = np.isnan(t)
    sat = (~nan) & (t >= E4M3_MAX)
    sub = (~nan) & (t < _SUBNORMAL_LIMIT)
    nrm = ~(nan | sat | sub)

    # Subnormal range: value = m * 2^-9 with m = rne(t / 2^-9) in [0, 8];
    # m == 8 is exactly the smallest normal, whose code is also 8.
    out[sub] = np.rint(t[sub] / _SUBNORMAL_STEP).astype(np.int64)

    # Normal range: t = f * 2^ex with f in [0.5, 1) (frexp), so the unbiased
    # E4M3 exponent is e = ex - 1 and t / 2^e lies in [1, 2).
    tn = t[nrm]
    _, ex = np.frexp(tn)
    e = ex.astype(np.int64) - 1
    frac = np.rint((np.ldexp(tn, -e) - 1.0) * 8.0).astype(np.int64)
    carry = frac == 8                     # rounded up to the next binade
    e = e + carry
    frac = np.where(carry, 0, frac)
    code = ((e + 7) << 3) | frac
    out[nrm] = np.minimum(code, _MAX_CODE)

    out[sat] = _MAX_CODE
    out[nan] = 0x7F
    out = out | (neg.astype(np.int64) << 7)
    return out.astype(np.uint8)
