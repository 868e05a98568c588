"""Seeded synthetic inputs for the FP8 W8A8 linear path.

This module draws random numbers and arranges them into the shapes of the
workloads; it holds none of the quantization, GEMM or dequantization
arithmetic.  Both the CUDA path and the CPU oracle are fed from here, so the
two always see the same bytes.

Workloads (shapes and distributions follow the FP8 serving description of
OneRec-V2: per-token activations with a few outlier channels, LLM-style weight
init, a fat MoE with top-2 routing and FP16 router logits):

  tiny     X [32,256] ~ N(0,1)                 W [256,256]  ~ N(0, 0.02^2)
  qkv      X [4096,2048] ~ N(0,1), 1% channels x50    W [6144,2048]
  ffn_up   X [8192,2048], 0.5% channels x30           W1 [8192,2048]
  ffn_down X [8192,8192], 0.5% channels x30           W2 [2048,8192]
  moe      X [8192,2048] ~ N(0,1); logits fp16 [8192,64] ~ N(0,1) -> top-2
           W_up [64,1024,2048], W_down [64,2048,1024]
  sweep    X [M,4096] with |x| = exp(N(0,1)) and random signs; W [4096,4096]

Seeds: workload i (0-based, in the order above, ffn_up/ffn_down sharing one)
draws X from seed i, W from seed 100+i and outlier channels / router logits
from seed 200+i.  Everything is generated on the CPU in float32 and cast to
float16, so results do not depend on the device.

Source pages: "Quantized Inference for OneRec-V2" (section 关键证据: per-channel
weights, per-token activations, QKV/O, dense FFN and MoE grouped GEMM) and
"FP8量化在生成式推荐系统OneRec-V2中的优化实践" (§1.2 numeric profile: weight
variance ~1e-1, activation maxima ~1e2; §2.1 merged QKV; §3.2 MoE).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

W_STD = 0.02
SWEEP_M = (1, 8, 32, 128, 512, 2048, 8192, 16384)
SWEEP_K = 4096
SWEEP_N = 4096
MOE_T, MOE_D, MOE_E, MOE_TOPK, MOE_F = 8192, 2048, 64, 2, 1024


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def normal_f16(shape, std: float, g: torch.Generator) -> torch.Tensor:
    """N(0, std^2) drawn in float32 and rounded to float16."""
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * std).to(torch.float16)


def with_outlier_channels(x32: torch.Tensor, n_channels: int, factor: float,
                          g: torch.Generator) -> torch.Tensor:
    """Scale `n_channels` randomly chosen columns of a float32 matrix by `factor`."""
    k = x32.shape[1]
    ch = torch.randperm(k, generator=g)[:n_channels]
    x32[:, ch] *= factor
    return x32


@dataclass
class Linear:
    name: str
    X: torch.Tensor      # fp16 [M,K]
    W: torch.Tensor      # fp16 [N,K]


def tiny() -> Linear:
    X = normal_f16((32, 256), 1.0, _gen(0))
    W = normal_f16((256, 256), W_STD, _gen(100))
    return Linear("tiny", X, W)


def qkv(m: int = 4096) -> Linear:
    """Merged QKV projection: 32 requests x 128 beam tokens, d=2048, N=3*2048."""
    K, N = 2048, 6144
    x = torch.randn(m, K, generator=_gen(1), dtype=torch.float32)
    x = with_outlier_channels(x, 20, 50.0, _gen(201))
    W = normal_f16((N, K), W_STD, _gen(101))
    return Linear("qkv", x.to(torch.float16), W)


def ffn() -> tuple[Linear, Linear]:
    """Dense FFN pair; up and down inputs are drawn independently (not chained)."""
    gx, gw, go = _gen(2), _gen(102), _gen(202)
    xu = torch.randn(8192, 2048, generator=gx, dtype=torch.float32)
    xd = torch.randn(8192, 8192, generator=gx, dtype=torch.float32)
    W1 = normal_f16((8192, 2048), W_STD, gw)
    W2 = normal_f16((2048, 8192), W_STD, gw)
    xu = with_outlier_channels(xu, 10, 30.0, go)
    xd = with_outlier_channels(xd, 41, 30.0, go)
    return (Linear("ffn_up", xu.to(torch.float16), W1),
            Linear("ffn_down", xd.to(torch.float16), W2))


def sweep_x(m: int) -> torch.Tensor:
    """Lognormal-magnitude activations with random signs, [m, 4096]."""
    g = _gen(4)
    mag = torch.exp(torch.randn(m, SWEEP_K, generator=g, dtype=torch.float32))
    sign = torch.randint(0, 2, (m, SWEEP_K), generator=g, dtype=torch.int8).to(torch.float32) * 2 - 1
    return (mag * sign).to(torch.float16)


def sweep_w() -> torch.Tensor:
    return normal_f16((SWEEP_N, SWEEP_K), W_STD, _gen(104))


def sweep(m: int) -> Linear:
    return Linear(f"sweep_m{m}", sweep_x(m), sweep_w())


# ---------------------------------------------------------------------------
# MoE: FP16 router (harness only, not on the FP8 path) and expert grouping.
# ---------------------------------------------------------------------------

def route_top2(logits_f16: np.ndarray, topk: int = MOE_TOPK) -> np.ndarray:
    """Top-k experts per token from FP16 gate logits.

    Highest logit first; equal logits go to the lower expert id (a stable sort
    of the negated logits keeps the lower index first among ties).
    Returns int64 [T, topk].
    """
    neg = -logits_f16.astype(np.float32)
    return np.argsort(neg, axis=1, kind="stable")[:, :topk].astype(np.int64)


def _expert_order(experts: np.ndarray) -> np.ndarray:
    """Permutation of the flattened (token, slot) pairs that sorts them by (expert, token)."""
    T, k = experts.shape
    tok = np.repeat(np.arange(T, dtype=np.int64), k)
    return np.lexsort((tok, experts.reshape(-1)))


def group_by_expert(experts: np.ndarray, n_experts: int) -> tuple[np.ndarray, np.ndarray]:
    """Order (token, slot) pairs by (expert, token).

    Returns (token_of_row int64 [T*topk], offsets int32 [E+1]) where rows
    offsets[e]..offsets[e+1] hold the tokens routed to expert e, ascending.
    """
    T, k = experts.shape
    tok = np.repeat(np.arange(T, dtype=np.int64), k)
    order = _expert_order(experts)
    counts = np.bincount(experts.reshape(-1), minlength=n_experts)
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    np.cumsum(counts, out=offsets[1:])
    return tok[order], offsets.astype(np.int32)


def gate_weights(logits_f16: np.ndarray, experts: np.ndarray) -> np.ndarray:
    """Combine weights of each token's selected experts: a softmax over the
    selected FP16 logits, in float32 (harness side of the router; the pages
    fix no combine rule).  Returns float32 [T, topk], rows summing to ~1."""
    sel = np.take_along_axis(logits_f16.astype(np.float32), experts, axis=1)
    z = np.exp(sel - sel.max(axis=1, keepdims=True), dtype=np.float32)
    return (z / z.sum(axis=1, keepdims=True)).astype(np.float32)


def token_rows(row_token: np.ndarray, tokens: int, topk: int = MOE_TOPK) -> np.ndarray:
    """Inverse of the grouping: int32 [tokens, topk], the grouped rows of each
    token in row order (-1 where a token has fewer than topk rows)."""
    out = np.full((tokens, topk), -1, dtype=np.int32)
    fill = np.zeros(tokens, dtype=np.int64)
    for r, t in enumerate(np.asarray(row_token, dtype=np.int64)):
        if fill[t] >= topk:
            raise ValueError(f"token {t} has more than {topk} rows")
        out[t, fill[t]] = r
        fill[t] += 1
    return out


def row_weights(weights: np.ndarray, experts: np.ndarray) -> np.ndarray:
    """The combine weight of every grouped row (same order as group_by_expert): float32 [T*topk]."""
    return weights.reshape(-1)[_expert_order(experts)].astype(np.float32)


@dataclass
class MoE:
    X: torch.Tensor          # fp16 [T, d]   tokens in arrival order
    logits: torch.Tensor     # fp16 [T, E]
    token_of_row: np.ndarray  # int64 [T*topk]
    offsets: np.ndarray      # int32 [E+1]
    X_perm: torch.Tensor     # fp16 [T*topk, d] rows in expert order
    W_up: torch.Tensor       # fp16 [E, F, d]
    W_down: torch.Tensor     # fp16 [E, d, F]
    row_weight: np.ndarray   # float32 [T*topk] combine weight of each grouped row (see gate_weights)


def moe(T: int = MOE_T, d: int = MOE_D, E: int = MOE_E, F: int = MOE_F,
        with_weights: bool = True) -> MoE:
    X = normal_f16((T, d), 1.0, _gen(3))
    logits = normal_f16((T, E), 1.0, _gen(203))
    experts = route_top2(logits.numpy())
    token_of_row, offsets = group_by_expert(experts, E)
    X_perm = X[torch.from_numpy(token_of_row)]
    if with_weights:
        gw = _gen(103)
        W_up = normal_f16((E, F, d), W_STD, gw)
        W_down = normal_f16((E, d, F), W_STD, gw)
    else:
        W_up = W_down = None
    row_weight = row_weights(gate_weights(logits.numpy(), experts), experts)
    return MoE(X, logits, token_of_row, offsets, X_perm, W_up, W_down, row_weight)


def offsets_from_counts(counts) -> np.ndarray:
    counts = np.asarray(counts, dtype=np.int64)
    off = np.zeros(len(counts) + 1, dtype=np.int64)
    np.cumsum(counts, out=off[1:])
    return off.astype(np.int32)


def random_f16(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    """Generic seeded N(0,std^2) fp16 tensor for edge-case tests."""
    return normal_f16(shape, std, _gen(seed))
