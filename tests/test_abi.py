"""The C ABI library loads, exports every symbol declared in include/fp8q.h,
and rejects bad arguments on the host before touching the GPU (no GPU needed)."""
import os
import re

import pytest

from fp8_quantized_generative_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8q.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8q_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(_lib.LIB_PATH):
        from fp8_quantized_generative_b200 import build
        build.build()
    return _lib.lib()


def test_header_declares_the_path_entry_points():
    names = declared_functions()
    for required in ("fp8q_quantize_weight_per_channel", "fp8q_quantize_rows_dynamic", "fp8q_linear",
                     "fp8q_moe_grouped_linear"):
        assert required in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_status_strings(L):
    assert _lib.status_string(0) == "FP8Q_OK"
    assert _lib.status_string(1) == "FP8Q_ERR_INVALID_ARG"
    assert _lib.status_string(99) == "FP8Q_UNKNOWN_STATUS"
    assert L.fp8q_version() >= 100


BAD = 0x1008   # 8-byte aligned, not 16


@pytest.mark.parametrize("args", [
    (0, 4, 32, 0x1000, 0x2000, 0),          # null X
    (0x1000, 4, 32, 0, 0x2000, 0),          # null Xq
    (0x1000, -1, 32, 0x1000, 0x2000, 0),    # negative M
    (0x1000, 4, 0, 0x1000, 0x2000, 0),      # K = 0
    (0x1000, 4, 24, 0x1000, 0x2000, 0),     # K % 16 != 0
    (BAD, 4, 32, 0x1000, 0x2000, 0),        # misaligned
])
def test_quantize_rejects(L, args):
    assert _lib.fp8q_quantize_rows_dynamic(*args) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.last_error_message() != ""


def test_quantize_zero_rows_is_noop(L):
    assert _lib.fp8q_quantize_rows_dynamic(0, 0, 32, 0, 0, 0) == _lib.FP8Q_OK
    assert _lib.fp8q_quantize_weight_per_channel(0, 0, 32, 0, 0, 0) == _lib.FP8Q_ERR_INVALID_ARG


@pytest.mark.parametrize("M,N,K,ptrs", [
    (4, 0, 32, None), (4, 12, 32, None), (4, 16, 40, None), (-2, 16, 32, None),
    (4, 16, 32, (0, 0x1000, 0x1000, 0x1000, 0x1000)),
    (4, 16, 32, (0x1000, 0x1000, BAD, 0x1000, 0x1000)),
])
def test_linear_rejects(L, M, N, K, ptrs):
    p = ptrs or (0x1000,) * 5
    assert _lib.fp8q_linear(p[0], p[1], p[2], p[3], M, N, K, p[4], 0) == _lib.FP8Q_ERR_INVALID_ARG


def test_linear_zero_rows_is_noop(L):
    assert _lib.fp8q_linear(0, 0, 0, 0, 0, 16, 32, 0, 0) == _lib.FP8Q_OK


@pytest.mark.parametrize("E,rows,N,K,off", [
    (0, 8, 16, 32, 0x1000), (1025, 8, 16, 32, 0x1000), (4, 8, 12, 32, 0x1000),
    (4, 8, 16, 20, 0x1000), (4, 8, 16, 32, 0), (4, 8, 16, 32, 0x1002), (4, -1, 16, 32, 0x1000),
])
def test_moe_rejects(L, E, rows, N, K, off):
    a = 0x1000
    assert _lib.fp8q_moe_grouped_linear(a, a, off, E, rows, a, a, N, K, a, 0) == _lib.FP8Q_ERR_INVALID_ARG


def test_encode_rejects(L):
    assert _lib.fp8q_e4m3_encode_f32(0, 10, 0x1000, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_e4m3_encode_f32(0x1000, -1, 0x1000, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_e4m3_encode_f32(0, 0, 0, 0) == _lib.FP8Q_OK


def test_python_wrappers_refuse_cpu_tensors():
    import torch
    import fp8_quantized_generative_b200 as fq
    with pytest.raises(ValueError):
        fq.quantize_rows_dynamic(torch.zeros(4, 32, dtype=torch.float16))


def test_selftest_rejects_bad_limits(L):
    assert _lib.fp8q_selftest_wait_timeout(0, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_selftest_wait_timeout(3_000_000, 0) == _lib.FP8Q_ERR_INVALID_ARG


@pytest.mark.parametrize("M,N,K,ws", [
    (-1, 16, 32, (0, 0)), (4, 12, 32, (0, 0)), (4, 16, 24, (0, 0)),
    (4, 16, 32, (0x1000, 0)), (4, 16, 32, (0x1008, 0x1000)),
])
def test_quantized_linear_rejects(L, M, N, K, ws):
    a = 0x1000
    assert _lib.fp8q_quantized_linear(a, a, a, M, N, K, a, ws[0], ws[1], 0) == _lib.FP8Q_ERR_INVALID_ARG


def test_quantized_linear_zero_rows_noop(L):
    assert _lib.fp8q_quantized_linear(0, 0, 0, 0, 16, 32, 0, 0, 0, 0) == _lib.FP8Q_OK


def test_format_variants_reject_bad_format_and_shapes(L):
    a = 0x1000
    # unknown format codes are refused before anything runs
    assert _lib.fp8q_quantize_rows_dynamic_fmt(a, 4, 32, 2, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_quantize_rows_dynamic_fmt(a, 4, 32, -1, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_linear_fmt(a, 2, a, a, a, 4, 16, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_moe_grouped_linear_fmt(a, 7, a, a, 4, 8, a, a, 16, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    # valid format, bad shapes or pointers
    assert _lib.fp8q_quantize_rows_dynamic_fmt(a, 4, 24, _lib.FP8Q_FMT_E5M2, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_quantize_rows_dynamic_fmt(a, 0, 32, _lib.FP8Q_FMT_E5M2, 0, 0, 0) == _lib.FP8Q_OK
    assert _lib.fp8q_linear_fmt(a, _lib.FP8Q_FMT_E5M2, a, BAD, a, 4, 16, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_linear_fmt(0, _lib.FP8Q_FMT_E5M2, 0, 0, 0, 0, 16, 32, 0, 0) == _lib.FP8Q_OK
    assert _lib.fp8q_moe_grouped_linear_fmt(a, _lib.FP8Q_FMT_E5M2, a, a, 0, 8, a, a, 16, 32, a, 0) \
        == _lib.FP8Q_ERR_INVALID_ARG


def test_per_tensor_rejects(L):
    a = 0x1000
    assert _lib.fp8q_quantize_weight_per_tensor(a, 0, 32, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_quantize_weight_per_tensor(a, 4, 40, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_quantize_weight_per_tensor(BAD, 4, 32, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_quantize_weight_per_tensor(a, 4, 32, a, 0, 0) == _lib.FP8Q_ERR_INVALID_ARG


def test_blockscaled_rejects(L):
    a = 0x1000
    assert _lib.fp8q_quantize_weight_blockwise(a, 0, 16, 32, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_quantize_weight_blockwise(a, 2, 0, 32, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_quantize_weight_blockwise(a, 2, 16, 40, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert _lib.fp8q_quantize_weight_blockwise(BAD, 2, 16, 32, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    mo = _lib.fp8q_moe_grouped_linear_blockscaled
    assert mo(a, a, a, 129, 8, a, a, 16, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG      # E > 128
    assert mo(a, a, a, 0, 8, a, a, 16, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert mo(a, a, a, 4, 8, a, a, 12, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG       # N % 8
    assert mo(a, a, a, 4, 8, a, a, 16, 24, a, 0) == _lib.FP8Q_ERR_INVALID_ARG       # K % 16
    assert mo(a, a, 0x1002, 4, 8, a, a, 16, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG  # offsets alignment
    assert mo(a, a, a, 4, 8, a, BAD, 16, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert mo(0, 0, a, 4, 0, 0, 0, 16, 32, 0, 0) == _lib.FP8Q_OK                    # no rows


def test_gather_rejects(L):
    a = 0x1000
    g = _lib.fp8q_moe_grouped_linear_gather
    assert g(a, a, 0, a, a, 4, 8, a, a, 16, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG      # no tokens
    assert g(a, a, 10, 0, a, 4, 8, a, a, 16, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG     # null row_token
    assert g(a, a, 10, 0x1002, a, 4, 8, a, a, 16, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert g(a, a, 10, a, a, 0, 8, a, a, 16, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert g(a, a, 10, a, a, 4, 8, a, a, 12, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert g(BAD, a, 10, a, a, 4, 8, a, a, 16, 32, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert g(0, 0, 10, a, a, 4, 0, 0, 0, 16, 32, 0, 0) == _lib.FP8Q_OK                  # no rows


def test_combine_rejects(L):
    a = 0x1000
    c = _lib.fp8q_moe_grouped_linear_combine
    #      Xq s_x off E  rows Wq s_w N   K  tok w  T   out st
    assert c(a, a, a, 4, 8, a, a, 16, 32, a, a, 0, a, 0) == _lib.FP8Q_ERR_INVALID_ARG     # no tokens
    assert c(a, a, a, 0, 8, a, a, 16, 32, a, a, 4, a, 0) == _lib.FP8Q_ERR_INVALID_ARG     # E = 0
    assert c(a, a, a, 4, 8, a, a, 12, 32, a, a, 4, a, 0) == _lib.FP8Q_ERR_INVALID_ARG     # N % 8
    assert c(a, a, a, 4, 8, a, a, 16, 24, a, a, 4, a, 0) == _lib.FP8Q_ERR_INVALID_ARG     # K % 16
    assert c(a, a, a, 4, 8, a, a, 16, 32, 0, a, 4, a, 0) == _lib.FP8Q_ERR_INVALID_ARG     # null row_token
    assert c(a, a, a, 4, 8, a, a, 16, 32, a, 0x1002, 4, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert c(a, a, a, 4, 8, a, a, 16, 32, a, a, 4, BAD, 0) == _lib.FP8Q_ERR_INVALID_ARG   # output alignment
    assert c(a, a, 0x1002, 4, 8, a, a, 16, 32, a, a, 4, a, 0) == _lib.FP8Q_ERR_INVALID_ARG


def test_dispatch_rejects(L):
    a = 0x1000
    d = _lib.fp8q_quantize_rows_dispatch
    #      X  T   K   fmt tr topk rows Xq s  st
    assert d(a, 4, 32, 0, a, 0, 8, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG      # topk 0
    assert d(a, 4, 32, 0, a, 9, 8, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG      # topk > 8
    assert d(a, 4, 32, 2, a, 2, 8, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG      # fmt
    assert d(a, 4, 24, 0, a, 2, 8, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG      # K % 16
    assert d(a, 4, 32, 0, 0, 2, 8, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG      # null token_rows
    assert d(a, 4, 32, 0, 0x1002, 2, 8, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert d(a, 4, 32, 0, a, 2, 8, BAD, a, 0) == _lib.FP8Q_ERR_INVALID_ARG    # Xq alignment
    assert d(a, 4, 32, 0, a, 2, 0, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG      # tokens, no rows
    assert d(0, 0, 32, 0, 0, 2, 0, 0, 0, 0) == _lib.FP8Q_OK                   # nothing to do


def test_overlapped_rejects_and_sync_words(L):
    a = 0x1000
    o = _lib.fp8q_quantized_linear_overlapped
    #      X  Wq sw M    N   K   Y  Xq sx sync st
    assert o(a, a, a, 300, 12, 32, a, a, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG     # N % 8
    assert o(a, a, a, 300, 16, 24, a, a, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG     # K % 16
    assert o(a, a, a, 300, 16, 32, a, a, a, 0, 0) == _lib.FP8Q_ERR_INVALID_ARG     # null sync
    assert o(a, a, a, 300, 16, 32, a, a, a, BAD, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert o(a, a, a, 300, 16, 32, a, BAD, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert o(a, a, a, -1, 16, 32, a, a, a, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert o(0, 0, 0, 0, 16, 32, 0, 0, 0, 0, 0) == _lib.FP8Q_OK                     # M = 0
    w = _lib.fp8q_overlap_sync_words
    assert [w(0), w(1), w(128), w(129), w(4096)] == [2, 4, 4, 6, 66]


def test_combine_rejects_misaligned_operands_before_touching_the_output(L):
    # with rows > 0, a misaligned operand is rejected on the host (no memset is queued)
    a = 0x1000
    c = _lib.fp8q_moe_grouped_linear_combine
    assert c(BAD, a, a, 4, 8, a, a, 16, 32, a, a, 4, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
    assert c(a, a, a, 4, 8, BAD, a, 16, 32, a, a, 4, a, 0) == _lib.FP8Q_ERR_INVALID_ARG
