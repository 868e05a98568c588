"""Per-row dynamic quantization to E4M3 with one fp32 scale per row.

Used for both granularities on the path [P1 关键证据, steps 1-2]:
  * weights W[N,K], one scale per output channel (row), computed offline;
  * activations X[M,K], one scale per token (row), computed at run time.

Per row (reading of [P2 §2.2], whose sample computes the scale as
max_code / max(|x|, eps) and divides to dequantize; here max_code = 448, the
E4M3 maximum of [P2 §1.2]):
    a  = max_k |A[k]|                     (exact in float32)
    a' = max(a, eps),  eps = 1e-12        (all-zero rows stay finite)
    r  = fl32(448 / a')                   (one IEEE fp32 division, RN)
    s  = fl32(a' / 448)                   (one IEEE fp32 division, RN; stored)
    q[k] = E4M3_rne_sat( fl32(A[k] * r) ) (one fp32 multiply, RN, then encode)
Dequantization is q * s.  NumPy float32 division and multiplication are the
IEEE round-to-nearest operations, so these are exactly the fp32 steps stated.
"""
from __future__ import annotations

import numpy as np

from .e4m3 import E4M3_MAX, e4m3_encode

EPS = np.float32(1e-12)


def quant_rows(A) -> tuple[np.ndarray, np.ndarray]:
    """A: float16 (or float32) [R, K] -> (codes uint8 [R, K], scales float32 [R])."""
    a32 = np.asarray(A).astype(np.float32)
    if a32.ndim != 2:
        raise ValueError("quant_rows expects a 2-D matrix")
    if a32.shape[1] == 0:
        amax = np.zeros(a32.shape[0], dtype=np.float32)
    else:
        amax = np.max(np.abs(a32), axis=1)
    amax = np.maximum(amax, EPS).astype(np.float32)
    qmax = np.float32(E4M3_MAX)
    r = (qmax / amax).astype(np.float32)
    s = (amax / qmax).astype(np.float32)
    prod = (a32 * r[:, None]).astype(np.float32)
    return e4m3_encode(prod), s
