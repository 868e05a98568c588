"""B200-native FP8 W8A8 linear layers (per-channel weights, per-token
dynamic activations, FP8 tensor-core GEMM with FP32 accumulation and a fused
dequantize + FP16 epilogue; dense and MoE grouped).

The compute runs in libfp8q.so (hand-written sm_100a kernels behind a C ABI,
include/fp8q.h).  This module only marshals torch tensors into that ABI:
PyTorch provides device memory and streams.  There is no CPU fallback; a
missing library raises ImportError at the first call.

    Xq, s_x = quantize_rows_dynamic(X)          # X fp16 [M,K] on cuda
    Wq, s_w = quantize_weight_per_channel(W)    # offline, W fp16 [N,K]
    Y = linear(Xq, s_x, Wq, s_w)                # fp16 [M,N]
    Y = moe_grouped_linear(Xq, s_x, offsets, Wq_e, s_w_e)

Variants from the pages: activations in E5M2 (quantize_rows_dynamic(X,
fmt="e5m2") with linear(..., x_fmt="e5m2")), per-tensor weight scales
(quantize_weight_per_tensor) and 128x128 block-scaled MoE expert weights
(quantize_weight_blockwise with moe_grouped_linear_blockscaled).
"""
from __future__ import annotations

import torch

from . import _lib
from ._lib import Fp8qError, check, lib

__all__ = [
    "Fp8qError", "lib", "quantize_rows_dynamic", "quantize_weight_per_channel", "quantize_weight_per_tensor",
    "quantize_weight_blockwise", "linear", "moe_grouped_linear", "moe_grouped_linear_gather",
    "moe_grouped_linear_combine", "quantize_rows_dispatch", "quantized_linear_overlapped", "overlap_workspace",
    "moe_grouped_linear_blockscaled",
    "quantized_linear", "e4m3_encode_f32", "device_error", "set_gemm_tuning",
]


def _fmt(name: str) -> int:
    try:
        return _lib.FORMATS[name]
    except KeyError:
        raise ValueError(f"unknown FP8 format {name!r} (e4m3 or e5m2)") from None


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _need(t: torch.Tensor, dtype, name: str, ndim: int | None = None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D, got shape {tuple(t.shape)}")


def quantize_rows_dynamic(X: torch.Tensor, out: tuple | None = None, fmt: str = "e4m3"):
    """Per-token dynamic FP8 quantization: fp16 [M,K] -> (uint8 [M,K], fp32 [M]).
    fmt: "e4m3" (the path) or "e5m2" (the activation-format variant)."""
    _need(X, torch.float16, "X", 2)
    M, K = X.shape
    Xq, s = out if out is not None else (
        torch.empty((M, K), dtype=torch.uint8, device=X.device),
        torch.empty((M,), dtype=torch.float32, device=X.device))
    if fmt == "e4m3":
        check(_lib.fp8q_quantize_rows_dynamic(X.data_ptr(), M, K, Xq.data_ptr(), s.data_ptr(), _stream(X)),
              "fp8q_quantize_rows_dynamic")
    else:
        check(_lib.fp8q_quantize_rows_dynamic_fmt(X.data_ptr(), M, K, _fmt(fmt), Xq.data_ptr(), s.data_ptr(),
                                                  _stream(X)), "fp8q_quantize_rows_dynamic_fmt")
    return Xq, s


def quantize_rows_dispatch(X: torch.Tensor, token_rows: torch.Tensor, rows: int, out: tuple | None = None,
                           fmt: str = "e4m3"):
    """Per-token quantization of X fp16 [T,K] written to the expert-grouped
    rows: token t's codes and scale go to rows token_rows[t, j] (int32
    [T, topk], -1 = none) of the returned (uint8 [rows,K], fp32 [rows])."""
    _need(X, torch.float16, "X", 2)
    _need(token_rows, torch.int32, "token_rows", 2)
    T, K = X.shape
    if token_rows.shape[0] != T:
        raise ValueError("token_rows must be [T, topk]")
    Xq, s = out if out is not None else (
        torch.empty((rows, K), dtype=torch.uint8, device=X.device),
        torch.empty((rows,), dtype=torch.float32, device=X.device))
    check(_lib.fp8q_quantize_rows_dispatch(X.data_ptr(), T, K, _fmt(fmt), token_rows.data_ptr(), token_rows.shape[1],
                                           rows, Xq.data_ptr(), s.data_ptr(), _stream(X)),
          "fp8q_quantize_rows_dispatch")
    return Xq, s


def quantize_weight_per_channel(W: torch.Tensor, out: tuple | None = None):
    """Offline per-output-channel E4M3 quantization: fp16 [N,K] or [E,N,K]."""
    _need(W, torch.float16, "W")
    if W.dim() not in (2, 3):
        raise ValueError("W must be [N,K] or [E,N,K]")
    K = W.shape[-1]
    rows = W.numel() // K
    Wq, s = out if out is not None else (torch.empty(W.shape, dtype=torch.uint8, device=W.device),
                                         torch.empty(W.shape[:-1], dtype=torch.float32, device=W.device))
    check(_lib.fp8q_quantize_weight_per_channel(W.data_ptr(), rows, K, Wq.data_ptr(), s.data_ptr(), _stream(W)),
          "fp8q_quantize_weight_per_channel")
    return Wq, s


def quantize_weight_per_tensor(W: torch.Tensor):
    """Offline per-tensor E4M3 quantization of fp16 [N,K]: one scale for the
    matrix, returned replicated as fp32 [N] (the form linear() takes)."""
    _need(W, torch.float16, "W", 2)
    N, K = W.shape
    Wq = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    s = torch.empty((N,), dtype=torch.float32, device=W.device)
    check(_lib.fp8q_quantize_weight_per_tensor(W.data_ptr(), N, K, Wq.data_ptr(), s.data_ptr(), _stream(W)),
          "fp8q_quantize_weight_per_tensor")
    return Wq, s


def linear(Xq: torch.Tensor, s_x: torch.Tensor, Wq: torch.Tensor, s_w: torch.Tensor,
           out: torch.Tensor | None = None, x_fmt: str = "e4m3") -> torch.Tensor:
    """FP8 W8A8 linear with fused dequantization: fp16 [M,N].  x_fmt: the
    format of the activation codes Xq ("e4m3" or "e5m2"); weights are E4M3."""
    _need(Xq, torch.uint8, "Xq", 2)
    _need(Wq, torch.uint8, "Wq", 2)
    _need(s_x, torch.float32, "s_x", 1)
    _need(s_w, torch.float32, "s_w", 1)
    M, K = Xq.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K or s_x.shape[0] != M or s_w.shape[0] != N:
        raise ValueError("shape mismatch")
    Y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=Xq.device)
    if x_fmt == "e4m3":
        check(_lib.fp8q_linear(Xq.data_ptr(), s_x.data_ptr(), Wq.data_ptr(), s_w.data_ptr(), M, N, K, Y.data_ptr(),
                               _stream(Xq)), "fp8q_linear")
    else:
        check(_lib.fp8q_linear_fmt(Xq.data_ptr(), _fmt(x_fmt), s_x.data_ptr(), Wq.data_ptr(), s_w.data_ptr(), M, N, K,
                                   Y.data_ptr(), _stream(Xq)), "fp8q_linear_fmt")
    return Y


FUSED_MAX_ROWS = 64


def quantized_linear(X: torch.Tensor, Wq: torch.Tensor, s_w: torch.Tensor,
                     out: torch.Tensor | None = None, fused: bool = False) -> torch.Tensor:
    """fp16 activations in, fp16 out: per-token quantization + FP8 linear +
    dequantization.  fused=True runs one kernel (up to 64 rows, no workspace);
    otherwise the two steps through a workspace allocated here."""
    _need(X, torch.float16, "X", 2)
    _need(Wq, torch.uint8, "Wq", 2)
    _need(s_w, torch.float32, "s_w", 1)
    M, K = X.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K or s_w.shape[0] != N:
        raise ValueError("shape mismatch")
    Y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=X.device)
    if fused and M <= FUSED_MAX_ROWS:
        st = _lib.fp8q_quantized_linear(X.data_ptr(), Wq.data_ptr(), s_w.data_ptr(), M, N, K, Y.data_ptr(), 0, 0,
                                        _stream(X))
        if st == _lib.FP8Q_OK:
            return Y
    Xq = torch.empty((M, K), dtype=torch.uint8, device=X.device)
    s_x = torch.empty((M,), dtype=torch.float32, device=X.device)
    check(_lib.fp8q_quantized_linear(X.data_ptr(), Wq.data_ptr(), s_w.data_ptr(), M, N, K, Y.data_ptr(),
                                     Xq.data_ptr(), s_x.data_ptr(), _stream(X)), "fp8q_quantized_linear")
    return Y


def overlap_workspace(M: int, K: int, device) -> tuple:
    """Workspace of quantized_linear_overlapped for M rows of K: (codes uint8
    [M,K], scales fp32 [M], sync words int32, zero-filled).  Reusable across
    calls that do not overlap on the GPU."""
    words = int(_lib.fp8q_overlap_sync_words(M))
    return (torch.empty((M, K), dtype=torch.uint8, device=device),
            torch.empty((M,), dtype=torch.float32, device=device),
            torch.zeros((words,), dtype=torch.int32, device=device))


def quantized_linear_overlapped(X: torch.Tensor, Wq: torch.Tensor, s_w: torch.Tensor,
                                workspace: tuple | None = None, out: torch.Tensor | None = None) -> torch.Tensor:
    """quantized_linear as one kernel for M > 128: the GEMM's own warps
    quantize the rows while its tensor cores start on the rows already done.
    The workspace (see overlap_workspace) then holds the codes and scales."""
    _need(X, torch.float16, "X", 2)
    _need(Wq, torch.uint8, "Wq", 2)
    _need(s_w, torch.float32, "s_w", 1)
    M, K = X.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K or s_w.shape[0] != N:
        raise ValueError("shape mismatch")
    Xq, s_x, sync = workspace if workspace is not None else overlap_workspace(M, K, X.device)
    if tuple(Xq.shape) != (M, K) or s_x.shape[0] != M or sync.numel() < _lib.fp8q_overlap_sync_words(M):
        raise ValueError("workspace does not fit this X")
    Y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=X.device)
    check(_lib.fp8q_quantized_linear_overlapped(X.data_ptr(), Wq.data_ptr(), s_w.data_ptr(), M, N, K, Y.data_ptr(),
                                                Xq.data_ptr(), s_x.data_ptr(), sync.data_ptr(), _stream(X)),
          "fp8q_quantized_linear_overlapped")
    return Y


def moe_grouped_linear(Xq: torch.Tensor, s_x: torch.Tensor, offsets: torch.Tensor, Wq: torch.Tensor,
                       s_w: torch.Tensor, out: torch.Tensor | None = None, x_fmt: str = "e4m3") -> torch.Tensor:
    """Expert-grouped FP8 linear.  offsets: int32 [E+1] on the device; x_fmt
    the format of the activation codes ("e4m3" or "e5m2")."""
    _need(Xq, torch.uint8, "Xq", 2)
    _need(s_x, torch.float32, "s_x", 1)
    _need(offsets, torch.int32, "offsets", 1)
    _need(Wq, torch.uint8, "Wq", 3)
    _need(s_w, torch.float32, "s_w", 2)
    rows, K = Xq.shape
    E, N, K2 = Wq.shape
    if K2 != K or offsets.shape[0] != E + 1 or tuple(s_w.shape) != (E, N) or s_x.shape[0] != rows:
        raise ValueError("shape mismatch")
    Y = out if out is not None else torch.empty((rows, N), dtype=torch.float16, device=Xq.device)
    if x_fmt == "e4m3":
        check(_lib.fp8q_moe_grouped_linear(Xq.data_ptr(), s_x.data_ptr(), offsets.data_ptr(), E, rows, Wq.data_ptr(),
                                           s_w.data_ptr(), N, K, Y.data_ptr(), _stream(Xq)),
              "fp8q_moe_grouped_linear")
    else:
        check(_lib.fp8q_moe_grouped_linear_fmt(Xq.data_ptr(), _fmt(x_fmt), s_x.data_ptr(), offsets.data_ptr(), E, rows,
                                               Wq.data_ptr(), s_w.data_ptr(), N, K, Y.data_ptr(), _stream(Xq)),
              "fp8q_moe_grouped_linear_fmt")
    return Y


def moe_grouped_linear_gather(Xq_tok: torch.Tensor, s_x_tok: torch.Tensor, row_token: torch.Tensor,
                              offsets: torch.Tensor, Wq: torch.Tensor, s_w: torch.Tensor,
                              out: torch.Tensor | None = None) -> torch.Tensor:
    """Expert-grouped FP8 linear whose row r reads token row_token[r] of the
    per-token codes Xq_tok [T,K] (scales s_x_tok [T]); rows in expert order
    (offsets int32 [E+1]); returns fp16 [len(row_token), N]."""
    _need(Xq_tok, torch.uint8, "Xq_tok", 2)
    _need(s_x_tok, torch.float32, "s_x_tok", 1)
    _need(row_token, torch.int32, "row_token", 1)
    _need(offsets, torch.int32, "offsets", 1)
    _need(Wq, torch.uint8, "Wq", 3)
    _need(s_w, torch.float32, "s_w", 2)
    T, K = Xq_tok.shape
    rows = row_token.shape[0]
    E, N, K2 = Wq.shape
    if K2 != K or offsets.shape[0] != E + 1 or tuple(s_w.shape) != (E, N) or s_x_tok.shape[0] != T:
        raise ValueError("shape mismatch")
    Y = out if out is not None else torch.empty((rows, N), dtype=torch.float16, device=Xq_tok.device)
    check(_lib.fp8q_moe_grouped_linear_gather(Xq_tok.data_ptr(), s_x_tok.data_ptr(), T, row_token.data_ptr(),
                                              offsets.data_ptr(), E, rows, Wq.data_ptr(), s_w.data_ptr(), N, K,
                                              Y.data_ptr(), _stream(Xq_tok)), "fp8q_moe_grouped_linear_gather")
    return Y


def moe_grouped_linear_combine(Xq: torch.Tensor, s_x: torch.Tensor, offsets: torch.Tensor, Wq: torch.Tensor,
                               s_w: torch.Tensor, row_token: torch.Tensor, row_weight: torch.Tensor, tokens: int,
                               out: torch.Tensor | None = None) -> torch.Tensor:
    """Expert-grouped FP8 linear whose row r is weighted by row_weight[r] and
    added (fp16) into row row_token[r] of the [tokens, N] output (the MoE
    down projection with the top-k combine)."""
    _need(Xq, torch.uint8, "Xq", 2)
    _need(s_x, torch.float32, "s_x", 1)
    _need(offsets, torch.int32, "offsets", 1)
    _need(Wq, torch.uint8, "Wq", 3)
    _need(s_w, torch.float32, "s_w", 2)
    _need(row_token, torch.int32, "row_token", 1)
    _need(row_weight, torch.float32, "row_weight", 1)
    rows, K = Xq.shape
    E, N, K2 = Wq.shape
    if (K2 != K or offsets.shape[0] != E + 1 or tuple(s_w.shape) != (E, N) or s_x.shape[0] != rows
            or row_token.shape[0] != rows or row_weight.shape[0] != rows):
        raise ValueError("shape mismatch")
    Y = out if out is not None else torch.empty((tokens, N), dtype=torch.float16, device=Xq.device)
    check(_lib.fp8q_moe_grouped_linear_combine(Xq.data_ptr(), s_x.data_ptr(), offsets.data_ptr(), E, rows,
                                               Wq.data_ptr(), s_w.data_ptr(), N, K, row_token.data_ptr(),
                                               row_weight.data_ptr(), tokens, Y.data_ptr(), _stream(Xq)),
          "fp8q_moe_grouped_linear_combine")
    return Y


BLOCK = 128


def quantize_weight_blockwise(W: torch.Tensor):
    """Offline 128x128 block-wise E4M3 quantization: fp16 [N,K] or [E,N,K] ->
    (uint8 same shape, fp32 scales [..., ceil(N/128), ceil(K/128)])."""
    _need(W, torch.float16, "W")
    if W.dim() not in (2, 3):
        raise ValueError("W must be [N,K] or [E,N,K]")
    E = W.shape[0] if W.dim() == 3 else 1
    N, K = W.shape[-2], W.shape[-1]
    Wq = torch.empty(W.shape, dtype=torch.uint8, device=W.device)
    s = torch.empty(W.shape[:-2] + (-(-N // BLOCK), -(-K // BLOCK)), dtype=torch.float32, device=W.device)
    check(_lib.fp8q_quantize_weight_blockwise(W.data_ptr(), E, N, K, Wq.data_ptr(), s.data_ptr(), _stream(W)),
          "fp8q_quantize_weight_blockwise")
    return Wq, s


def moe_grouped_linear_blockscaled(Xq: torch.Tensor, s_x: torch.Tensor, offsets: torch.Tensor, Wq: torch.Tensor,
                                   s_wb: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """Expert-grouped FP8 linear with 128x128 block-scaled expert weights
    (Wq [E,N,K] and s_wb [E, ceil(N/128), ceil(K/128)] from
    quantize_weight_blockwise); per-token activation scales."""
    _need(Xq, torch.uint8, "Xq", 2)
    _need(s_x, torch.float32, "s_x", 1)
    _need(offsets, torch.int32, "offsets", 1)
    _need(Wq, torch.uint8, "Wq", 3)
    _need(s_wb, torch.float32, "s_wb", 3)
    rows, K = Xq.shape
    E, N, K2 = Wq.shape
    if (K2 != K or offsets.shape[0] != E + 1 or s_x.shape[0] != rows
            or tuple(s_wb.shape) != (E, -(-N // BLOCK), -(-K // BLOCK))):
        raise ValueError("shape mismatch")
    Y = out if out is not None else torch.empty((rows, N), dtype=torch.float16, device=Xq.device)
    check(_lib.fp8q_moe_grouped_linear_blockscaled(Xq.data_ptr(), s_x.data_ptr(), offsets.data_ptr(), E, rows,
                                                   Wq.data_ptr(), s_wb.data_ptr(), N, K, Y.data_ptr(), _stream(Xq)),
          "fp8q_moe_grouped_linear_blockscaled")
    return Y


def e4m3_encode_f32(x: torch.Tensor) -> torch.Tensor:
    """The device E4M3 cast alone (diagnostic): fp32 -> uint8 codes."""
    _need(x, torch.float32, "x")
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    check(_lib.fp8q_e4m3_encode_f32(x.data_ptr(), x.numel(), out.data_ptr(), _stream(x)), "fp8q_e4m3_encode_f32")
    return out


def set_gemm_tuning(kernel_family: int = 0, tile_n: int = 0, ksplit: int = 0) -> None:
    """Override the dense-linear kernel choice (0 = automatic; see include/fp8q.h)."""
    check(_lib.fp8q_set_gemm_tuning(kernel_family, tile_n, ksplit), "fp8q_set_gemm_tuning")


def device_error(device=None) -> int:
    """Synchronize the current stream and return (and clear) the device error word."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st, flags = _lib.fp8q_device_error(torch.cuda.current_stream(dev).cuda_stream)
    if st not in (_lib.FP8Q_OK, _lib.FP8Q_ERR_TIMEOUT, _lib.FP8Q_ERR_DEVICE_CHECK):
        check(st, "fp8q_device_error")
    return flags
