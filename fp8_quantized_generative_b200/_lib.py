"""ctypes binding of libfp8q.so (the C ABI declared in include/fp8q.h).

Argument marshalling only: every entry point here forwards to the function
of the same name in the shared library.  Pointers are passed as integers
(device addresses), streams as integers (cudaStream_t handles).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8q.so")

FP8Q_OK = 0
FP8Q_ERR_INVALID_ARG = 1
FP8Q_ERR_UNSUPPORTED = 2
FP8Q_ERR_CUDA = 3
FP8Q_ERR_TIMEOUT = 4
FP8Q_ERR_DEVICE_CHECK = 5

FP8Q_FMT_E4M3 = 0
FP8Q_FMT_E5M2 = 1
FORMATS = {"e4m3": FP8Q_FMT_E4M3, "e5m2": FP8Q_FMT_E5M2}

DEVERR_TIMEOUT_PRODUCER = 0x1
DEVERR_TIMEOUT_MMA = 0x2
DEVERR_TIMEOUT_EPILOGUE = 0x4
DEVERR_BAD_OFFSETS = 0x8
DEVERR_TIMEOUT_CLUSTER = 0x10
DEVERR_TIMEOUT_SELFTEST = 0x20


class Fp8qError(RuntimeError):
    def __init__(self, status: int, what: str, message: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} {message}".rstrip())


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_INT = ctypes.c_int

# name -> (restype, argtypes); mirrors include/fp8q.h
SIGNATURES = {
    "fp8q_status_string": (ctypes.c_char_p, [_INT]),
    "fp8q_last_error_message": (ctypes.c_char_p, []),
    "fp8q_version": (_INT, []),
    "fp8q_quantize_rows_dynamic": (_INT, [_P, _I64, _I64, _P, _P, _P]),
    "fp8q_quantize_weight_per_channel": (_INT, [_P, _I64, _I64, _P, _P, _P]),
    "fp8q_linear": (_INT, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "fp8q_moe_grouped_linear": (_INT, [_P, _P, _P, _I32, _I64, _P, _P, _I64, _I64, _P, _P]),
    "fp8q_quantized_linear": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P]),
    "fp8q_quantized_linear_noalloc": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "fp8q_quantize_rows_dynamic_fmt": (_INT, [_P, _I64, _I64, _INT, _P, _P, _P]),
    "fp8q_quantize_weight_per_tensor": (_INT, [_P, _I64, _I64, _P, _P, _P]),
    "fp8q_linear_fmt": (_INT, [_P, _INT, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "fp8q_moe_grouped_linear_fmt": (_INT, [_P, _INT, _P, _P, _I32, _I64, _P, _P, _I64, _I64, _P, _P]),
    "fp8q_quantize_weight_blockwise": (_INT, [_P, _I32, _I64, _I64, _P, _P, _P]),
    "fp8q_quantized_linear_overlapped": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P]),
    "fp8q_overlap_sync_words": (_I64, [_I64]),
    "fp8q_quantize_rows_dispatch": (_INT, [_P, _I64, _I64, _I32, _P, _I32, _I64, _P, _P, _P]),
    "fp8q_moe_grouped_linear_combine": (_INT, [_P, _P, _P, _I32, _I64, _P, _P, _I64, _I64, _P, _P, _I64, _P, _P]),
    "fp8q_moe_grouped_linear_gather": (_INT, [_P, _P, _I64, _P, _P, _I32, _I64, _P, _P, _I64, _I64, _P, _P]),
    "fp8q_moe_grouped_linear_blockscaled": (_INT, [_P, _P, _P, _I32, _I64, _P, _P, _I64, _I64, _P, _P]),
    "fp8q_e4m3_encode_f32": (_INT, [_P, _I64, _P, _P]),
    "fp8q_set_gemm_tuning": (_INT, [_INT, _INT, _INT]),
    "fp8q_selftest_wait_timeout": (_INT, [ctypes.c_uint32, _P]),
    "fp8q_device_error": (_INT, [_P, ctypes.POINTER(ctypes.c_uint32)]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libfp8q.so once; fail loudly when it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"fp8q CUDA library missing: {LIB_PATH} — build it with "
                "`python -m fp8_quantized_generative_b200.build` (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    try:
        return lib().fp8q_status_string(int(status)).decode()
    except ImportError:
        return f"status {status}"


def last_error_message() -> str:
    return lib().fp8q_last_error_message().decode()


def check(status: int, what: str) -> None:
    if status != FP8Q_OK:
        raise Fp8qError(status, what, last_error_message())


# Raw entry points with the C names (integers in, status out).
def fp8q_quantize_rows_dynamic(X, M, K, Xq, s_x, stream):
    return lib().fp8q_quantize_rows_dynamic(X, M, K, Xq, s_x, stream)


def fp8q_quantize_weight_per_channel(W, N, K, Wq, s_w, stream):
    return lib().fp8q_quantize_weight_per_channel(W, N, K, Wq, s_w, stream)


def fp8q_linear(Xq, s_x, Wq, s_w, M, N, K, Y, stream):
    return lib().fp8q_linear(Xq, s_x, Wq, s_w, M, N, K, Y, stream)


def fp8q_quantized_linear(X, Wq, s_w, M, N, K, Y, Xq_ws, s_x_ws, stream):
    return lib().fp8q_quantized_linear(X, Wq, s_w, M, N, K, Y, Xq_ws, s_x_ws, stream)


def fp8q_quantized_linear_noalloc(X, Wq, s_w, M, N, K, Y, stream):
    return lib().fp8q_quantized_linear_noalloc(X, Wq, s_w, M, N, K, Y, stream)


def fp8q_moe_grouped_linear(Xq, s_x, offsets, E, rows, Wq, s_w, N, K, Y, stream):
    return lib().fp8q_moe_grouped_linear(Xq, s_x, offsets, E, rows, Wq, s_w, N, K, Y, stream)


def fp8q_quantize_rows_dynamic_fmt(X, M, K, fmt, Xq, s_x, stream):
    return lib().fp8q_quantize_rows_dynamic_fmt(X, M, K, fmt, Xq, s_x, stream)


def fp8q_quantize_weight_per_tensor(W, N, K, Wq, s_w, stream):
    return lib().fp8q_quantize_weight_per_tensor(W, N, K, Wq, s_w, stream)


def fp8q_linear_fmt(Xq, x_fmt, s_x, Wq, s_w, M, N, K, Y, stream):
    return lib().fp8q_linear_fmt(Xq, x_fmt, s_x, Wq, s_w, M, N, K, Y, stream)


def fp8q_moe_grouped_linear_fmt(Xq, x_fmt, s_x, offsets, E, rows, Wq, s_w, N, K, Y, stream):
    return lib().fp8q_moe_grouped_linear_fmt(Xq, x_fmt, s_x, offsets, E, rows, Wq, s_w, N, K, Y, stream)


def fp8q_moe_grouped_linear_gather(Xq_tok, s_x_tok, tokens, row_token, offsets, E, rows, Wq, s_w, N, K, Y, stream):
    return lib().fp8q_moe_grouped_linear_gather(Xq_tok, s_x_tok, tokens, row_token, offsets, E, rows, Wq, s_w, N, K,
                                                Y, stream)


def fp8q_quantized_linear_overlapped(X, Wq, s_w, M, N, K, Y, Xq_ws, s_x_ws, sync_ws, stream):
    return lib().fp8q_quantized_linear_overlapped(X, Wq, s_w, M, N, K, Y, Xq_ws, s_x_ws, sync_ws, stream)


def fp8q_overlap_sync_words(M):
    return lib().fp8q_overlap_sync_words(M)


def fp8q_quantize_rows_dispatch(X, T, K, fmt, token_rows, topk, rows, Xq, s_x, stream):
    return lib().fp8q_quantize_rows_dispatch(X, T, K, fmt, token_rows, topk, rows, Xq, s_x, stream)


def fp8q_moe_grouped_linear_combine(Xq, s_x, offsets, E, rows, Wq, s_w, N, K, row_token, row_weight, tokens, out,
                                    stream):
    return lib().fp8q_moe_grouped_linear_combine(Xq, s_x, offsets, E, rows, Wq, s_w, N, K, row_token, row_weight,
                                                 tokens, out, stream)


def fp8q_quantize_weight_blockwise(W, E, N, K, Wq, s_wb, stream):
    return lib().fp8q_quantize_weight_blockwise(W, E, N, K, Wq, s_wb, stream)


def fp8q_moe_grouped_linear_blockscaled(Xq, s_x, offsets, E, rows, Wq, s_wb, N, K, Y, stream):
    return lib().fp8q_moe_grouped_linear_blockscaled(Xq, s_x, offsets, E, rows, Wq, s_wb, N, K, Y, stream)


def fp8q_e4m3_encode_f32(x, n, out, stream):
    return lib().fp8q_e4m3_encode_f32(x, n, out, stream)


def fp8q_set_gemm_tuning(kernel_family, tile_n, ksplit=0):
    return lib().fp8q_set_gemm_tuning(kernel_family, tile_n, ksplit)


def fp8q_selftest_wait_timeout(limit_us, stream):
    return lib().fp8q_selftest_wait_timeout(limit_us, stream)


def fp8q_device_error(stream):
    flags = ctypes.c_uint32(0)
    st = lib().fp8q_device_error(stream, ctypes.byref(flags))
    return st, flags.value
