"""Per-row (and per-tensor) dynamic quantization to FP8 with fp32 scales.

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

Format variant ['FP8量化在生成式推荐系统OneRec-V2中的优化实践' §2.2: activations in
E5M2]: the same steps with max_code = 57344 (the E5M2 maximum) and the E5M2
encoder.

Per-tensor variant [same page, §2.1: the FFN linears use per-tensor
quantization; §2.2 keeps the activations per token, so the per-tensor scale
is the weight's]: a is the maximum over the whole matrix, then the same r, s
and codes; the one scale is returned replicated once per row (output
channel), the form the per-channel linear consumes.

Block-wise variant [same page, §2.1: the MoE expert grouped GEMM is
quantized "block-wise 128x128"; §2.2: block-aligned quantization for MoE]:
the weight matrix is cut into blocks of 128 output channels x 128 input
elements (ragged at the edges); each block gets its own a, r, s and codes
by the same steps; activations stay per token.
"""
from __future__ import annotations

import numpy as np

from .e4m3 import E4M3_MAX, e4m3_encode
from .e5m2 import E5M2_MAX, e5m2_encode

EPS = np.float32(1e-12)

# format name -> (largest finite code value, encoder)
FORMATS = {"e4m3": (E4M3_MAX, e4m3_encode), "e5m2": (E5M2_MAX, e5m2_encode)}


def _quant_with_amax(a32: np.ndarray, amax: np.ndarray, fmt: str) -> tuple[np.ndarray, np.ndarray]:
    """Codes and scales of rows a32 [R, K] given each row's amax [R]."""
    qmax_f, encode = FORMATS[fmt]
    amax = np.maximum(amax, EPS).astype(np.float32)
    qmax = np.float32(qmax_f)
    r = (qmax / amax).astype(np.float32)
    s = (amax / qmax).astype(np.float32)
    prod = (a32 * r[:, None]).astype(np.float32)
    return encode(prod), s


def quant_rows(A, fmt: str = "e4m3") -> tuple[np.ndarray, np.ndarray]:
    """A: float16 (or float32) [R, K] -> (codes uint8 [R, K], scales float32 [R])."""
    a32 = np.asarray(A).astype(np.float32)
    if a32.ndim != 2:
        raise ValueError("quant_rows expects a 2-D matrix")
    if a32.shape[1] == 0:
        amax = np.zeros(a32.shape[0], dtype=np.float32)
    else:
        amax = np.max(np.abs(a32), axis=1)
    return _quant_with_amax(a32, amax, fmt)


def quant_tensor(A) -> tuple[np.ndarray, np.ndarray]:
    """Per-tensor E4M3: one scale for the whole matrix A [R, K].

    Returns (codes uint8 [R, K], scales float32 [R]) with every scale equal.
    """
    a32 = np.asarray(A).astype(np.float32)
    if a32.ndim != 2:
        raise ValueError("quant_tensor expects a 2-D matrix")
    a = np.float32(np.max(np.abs(a32))) if a32.size else np.float32(0.0)
    return _quant_with_amax(a32, np.full(a32.shape[0], a, dtype=np.float32), "e4m3")


def quant_blocks(A, block: int = 128) -> tuple[np.ndarray, np.ndarray]:
    """Block-wise E4M3: A [R, K] -> (codes uint8 [R, K], scales float32 [ceil(R/b), ceil(K/b)]).

    Block (i, j) covers rows i*b .. i*b+b-1 and columns j*b .. j*b+b-1.
    """
    a32 = np.asarray(A).astype(np.float32)
    if a32.ndim != 2:
        raise ValueError("quant_blocks expects a 2-D matrix")
    R, K = a32.shape
    nb_r, nb_k = -(-R // block), -(-K // block)
    codes = np.zeros((R, K), dtype=np.uint8)
    scales = np.zeros((nb_r, nb_k), dtype=np.float32)
    for i in range(nb_r):
        for j in range(nb_k):
            blk = a32[i * block:(i + 1) * block, j * block:(j + 1) * block]
            a = np.float32(np.max(np.abs(blk))) if blk.size else np.float32(0.0)
            c, s = _quant_with_amax(blk, np.full(blk.shape[0], a, dtype=np.float32), "e4m3")
            codes[i * block:(i + 1) * block, j * block:(j + 1) * block] = c
            scales[i, j] = s[0] if s.size else np.float32(np.maximum(a, EPS) / np.float32(E4M3_MAX))
    return codes, scales
