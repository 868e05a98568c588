"""FP8 W8A8 linear and MoE grouped linear, double-accumulated.

[P1 关键证据, steps 3-4; P2 §2.3]: the matmul multiplies FP8 operands and
accumulates in at least FP32, then the result is brought back to FP16 before
the next layer; the dequantization uses the per-token scale s_x[m] and the
per-channel scale s_w[n].  Here the products and sums are taken in float64
(exact products, near-exact sums) so the oracle is at least as accurate as
any FP32 accumulation order:

    P[m,n] = sum_k dec(Xq[m,k]) * dec(Wq[n,k])          (float64)
    Y[m,n] = fp16_rne( (P[m,n] * s_x[m]) * s_w[n] )     (float64 -> float16)

With activations in E5M2 (['FP8量化在生成式推荐系统OneRec-V2中的优化实践'
§2.2]) only dec(Xq) changes: x_fmt names the activation codec.

Block-scaled weights (same page, §2.1, MoE: 128x128 blocks): each K block j
of 128 inputs contributes its partial product times the scale of the weight
block (n // 128, j):
    Y[m,n] = fp16_rne( s_x[m] * sum_j s_w[n // 128, j] * sum_{k in block j} dec(Xq[m,k]) * dec(Wq[n,k]) )
(float64 throughout).

No bias term (the pages name none).  The float64 -> float16 cast is NumPy's
direct, correctly rounded conversion (round half to even, overflow to inf).

MoE [P1 关键证据 item 2: the sparse MoE grouped GEMM]: rows are grouped by
expert, rows offsets[e]..offsets[e+1] use expert e's weights and scales.
"""
from __future__ import annotations

import numpy as np

from .e4m3 import e4m3_decode
from .e5m2 import e5m2_decode

_DECODERS = {"e4m3": e4m3_decode, "e5m2": e5m2_decode}


def _linear_f64(Xq, s_x, Wq, s_w, x_fmt: str = "e4m3") -> np.ndarray:
    """The dequantized product (P * s_x) * s_w in float64, before the fp16 cast."""
    Dx = _DECODERS[x_fmt](Xq)
    Dw = e4m3_decode(Wq)
    P = Dx @ Dw.T
    return (P * np.asarray(s_x, dtype=np.float64)[:, None]) * np.asarray(s_w, dtype=np.float64)[None, :]


def linear_ref(Xq, s_x, Wq, s_w, x_fmt: str = "e4m3") -> np.ndarray:
    """Xq uint8 [M,K], s_x f32 [M], Wq uint8 [N,K], s_w f32 [N] -> float16 [M,N]."""
    return _linear_f64(Xq, s_x, Wq, s_w, x_fmt).astype(np.float16)


def moe_ref(Xq, s_x, offsets, Wq, s_w, x_fmt: str = "e4m3") -> np.ndarray:
    """Grouped linear.

    Xq uint8 [R,K] (rows in expert order), s_x f32 [R], offsets int [E+1]
    with offsets[0] = 0 and offsets[E] = R, Wq uint8 [E,N,K], s_w f32 [E,N]
    -> float16 [R,N].  Empty groups produce no rows.
    """
    offsets = np.asarray(offsets, dtype=np.int64)
    E, N, _ = np.asarray(Wq).shape
    R = np.asarray(Xq).shape[0]
    if offsets.shape != (E + 1,) or offsets[0] != 0 or offsets[-1] != R or np.any(np.diff(offsets) < 0):
        raise ValueError("offsets must be non-decreasing, start at 0 and end at the row count")
    Y = np.zeros((R, N), dtype=np.float16)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            Y[lo:hi] = linear_ref(Xq[lo:hi], s_x[lo:hi], Wq[e], s_w[e], x_fmt)
    return Y


def linear_f64_unquantized(X, W) -> np.ndarray:
    """X @ W^T in float64 on the original (unquantized) values, for error-bound pins."""
    return np.asarray(X, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T


def linear_blockscaled_ref(Xq, s_x, Wq, s_wb, block: int = 128) -> np.ndarray:
    """Xq uint8 [M,K], s_x f32 [M], Wq uint8 [N,K], s_wb f32 [ceil(N/b), ceil(K/b)] -> float16 [M,N]."""
    Dx = e4m3_decode(Xq)
    Dw = e4m3_decode(Wq)
    M, K = Dx.shape
    N = Dw.shape[0]
    s_wb = np.asarray(s_wb, dtype=np.float64)
    acc = np.zeros((M, N))
    for j in range(-(-K // block)):
        part = Dx[:, j * block:(j + 1) * block] @ Dw[:, j * block:(j + 1) * block].T   # [M, N]
        col_scale = s_wb[np.arange(N) // block, j]                                        # [N]
        acc += part * col_scale[None, :]
    return (acc * np.asarray(s_x, dtype=np.float64)[:, None]).astype(np.float16)


def moe_blockscaled_ref(Xq, s_x, offsets, Wq, s_wb, block: int = 128) -> np.ndarray:
    """Grouped linear with block-scaled expert weights: Wq uint8 [E,N,K], s_wb f32 [E, ceil(N/b), ceil(K/b)]."""
    offsets = np.asarray(offsets, dtype=np.int64)
    E, N, _ = np.asarray(Wq).shape
    R = np.asarray(Xq).shape[0]
    if offsets.shape != (E + 1,) or offsets[0] != 0 or offsets[-1] != R or np.any(np.diff(offsets) < 0):
        raise ValueError("offsets must be non-decreasing, start at 0 and end at the row count")
    Y = np.zeros((R, N), dtype=np.float16)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            Y[lo:hi] = linear_blockscaled_ref(Xq[lo:hi], s_x[lo:hi], Wq[e], s_wb[e], block)
    return Y


def moe_gather_ref(Xq_tok, s_x_tok, row_token, offsets, Wq, s_w) -> np.ndarray:
    """Grouped linear whose rows are gathered from the token matrix.

    [P1 关键证据 item 2; P2 §3.2, inter-expert pipeline]: the routed rows of
    the MoE layer are the tokens themselves, so the activations are quantized
    once per token (Xq_tok uint8 [T,K], s_x_tok f32 [T]) and row r of the
    grouped product (rows in expert order, offsets as in moe_ref) reads token
    row_token[r].  Per-row quantization commutes with the row gather, so this
    equals moe_ref on the gathered (permuted) rows.
    """
    row_token = np.asarray(row_token, dtype=np.int64)
    Xq_tok = np.asarray(Xq_tok)
    if row_token.size and (row_token.min() < 0 or row_token.max() >= Xq_tok.shape[0]):
        raise ValueError("row_token out of range")
    return moe_ref(Xq_tok[row_token], np.asarray(s_x_tok)[row_token], offsets, Wq, s_w)


def moe_combine_ref(Xq, s_x, offsets, Wq, s_w, row_token, row_weight, tokens: int) -> np.ndarray:
    """Grouped linear whose rows are combined back into their tokens.

    The down projection of the MoE layer with the top-k combine in its
    epilogue [P1 关键证据 item 2; P2 §3.2]: each grouped row r (expert order,
    offsets as in moe_ref) yields y[r] = (P * s_x) * s_w in float64, its
    contribution c[r] = fp16(row_weight[r] * y[r]) (one rounding), and the
    output row of token t is the FP16 scatter-add of its contributions:
    out[t] starts at 0 and each contribution is added with one fp16 rounding
    of the exact sum.  With two rows per token (top-2) the result does not
    depend on the order of the additions (0 + a = a exactly and fp16
    addition is commutative).  Returns float16 [tokens, N].
    """
    offsets = np.asarray(offsets, dtype=np.int64)
    E, N, _ = np.asarray(Wq).shape
    R = np.asarray(Xq).shape[0]
    row_token = np.asarray(row_token, dtype=np.int64)
    w = np.asarray(row_weight, dtype=np.float32).astype(np.float64)
    if offsets.shape != (E + 1,) or offsets[0] != 0 or offsets[-1] != R or np.any(np.diff(offsets) < 0):
        raise ValueError("offsets must be non-decreasing, start at 0 and end at the row count")
    if row_token.shape != (R,) or (R and (row_token.min() < 0 or row_token.max() >= tokens)):
        raise ValueError("row_token out of range")
    out = np.zeros((tokens, N), dtype=np.float16)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        y = _linear_f64(Xq[lo:hi], s_x[lo:hi], Wq[e], s_w[e])
        c = (w[lo:hi, None] * y).astype(np.float16)
        for i, r in enumerate(range(lo, hi)):
            t = row_token[r]
            out[t] = (out[t].astype(np.float64) + c[i].astype(np.float64)).astype(np.float16)
    return out
