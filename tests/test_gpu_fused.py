"""GPU parity of the fused quantize + FP8 linear + dequantize path
(fp8q_quantized_linear): one kernel for up to 64 token rows (the CTAs of a
split-K cluster share the row maxima of their K slices), the two-step path
through a caller workspace above that."""
import numpy as np
import pytest
import torch

from fp8_quantized_generative_b200 import _lib
from fp8_quantized_generative_b200 import workloads as wl
from oracle import linear_ref, quant_rows

from parity import assert_close_f16, assert_no_device_error, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import fp8_quantized_generative_b200 as m
    assert torch.cuda.is_available()
    return m


def oracle(X, W):
    xq, sx = quant_rows(X.numpy())
    wq, sw = quant_rows(W.numpy())
    return linear_ref(xq, sx, wq, sw)


@pytest.mark.parametrize("M", [1, 5, 16, 17, 32, 33, 64])
@pytest.mark.parametrize("N,K", [(4096, 4096), (264, 272), (1000, 2048), (6144, 2048), (256, 16)])
def test_fused_against_oracle(fq, M, N, K):
    X = wl.random_f16((M, K), seed=M + N + K, std=2.0)
    W = wl.random_f16((N, K), seed=N * 3 + K, std=0.02)
    Wq, s_w = fq.quantize_weight_per_channel(W.cuda())
    Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    # the raw call without a workspace: it must take the one-kernel path
    Xd = X.cuda()
    st = _lib.fp8q_quantized_linear(Xd.data_ptr(), Wq.data_ptr(), s_w.data_ptr(), M, N, K, Y.data_ptr(), 0, 0,
                                    torch.cuda.current_stream().cuda_stream)
    assert st == _lib.FP8Q_OK, _lib.last_error_message()
    assert_close_f16(to_np(Y), oracle(X, W), f"fused {M}x{N}x{K}")
    Y2 = fq.quantized_linear(X.cuda(), Wq, s_w)        # two-step through a workspace
    assert_close_f16(to_np(Y2), oracle(X, W), f"two-step {M}x{N}x{K}")
    assert_no_device_error()


@pytest.mark.parametrize("ksplit", [1, 2, 4, 8])
@pytest.mark.parametrize("M", [7, 40, 64])
def test_fused_equals_two_step_bitwise(fq, ksplit, M):
    # Same split, same K range per CTA: the in-kernel quantization must give
    # exactly the quantizer kernel's codes and scales, hence identical output.
    # The two paths cut K into stages of different sizes (128 bytes fused,
    # 256 or 512 bytes for the workspace path), so K is chosen for every CTA
    # to get whole stages of each: a split of 8 takes K = 4096.
    N, K = 2048, (4096 if ksplit == 8 else 2048)
    X = wl.sweep_x(M)[:, :K].contiguous().cuda()
    Wq, s_w = fq.quantize_weight_per_channel(wl.random_f16((N, K), seed=5, std=0.02).cuda())
    fq.set_gemm_tuning(0, 0, ksplit)
    try:
        Yf = torch.empty((M, N), dtype=torch.float16, device="cuda")
        st = _lib.fp8q_quantized_linear(X.data_ptr(), Wq.data_ptr(), s_w.data_ptr(), M, N, K, Yf.data_ptr(), 0, 0,
                                        torch.cuda.current_stream().cuda_stream)
        assert st == _lib.FP8Q_OK, _lib.last_error_message()
        Xq, s_x = fq.quantize_rows_dynamic(X)
        Y2 = fq.linear(Xq, s_x, Wq, s_w)
    finally:
        fq.set_gemm_tuning(0, 0, 0)
    torch.cuda.synchronize()
    assert torch.equal(Yf, Y2)
    assert_no_device_error()


def test_edge_rows_fused(fq):
    K, N = 512, 256
    X = wl.random_f16((6, K), seed=9).float()
    X[0] = 0.0
    X[1, 3] = 65504.0
    X[2] = 2.0 ** -24
    X[3, ::2] = -0.0
    X = X.half()
    W = wl.random_f16((N, K), seed=10, std=0.02)
    Wq, s_w = fq.quantize_weight_per_channel(W.cuda())
    Y = fq.quantized_linear(X.cuda(), Wq, s_w, fused=True)
    y = to_np(Y)
    assert_close_f16(y, oracle(X, W), "fused edge rows")
    assert np.all(y[0] == 0)


def test_two_step_path_with_workspace(fq):
    M, N, K = 300, 520, 1040
    X = wl.random_f16((M, K), seed=1)
    W = wl.random_f16((N, K), seed=2, std=0.02)
    Wq, s_w = fq.quantize_weight_per_channel(W.cuda())
    Y = fq.quantized_linear(X.cuda(), Wq, s_w)
    assert_close_f16(to_np(Y), oracle(X, W), "two-step")
    # without a workspace the raw call refuses this shape
    Xd = X.cuda()
    Yd = torch.empty((M, N), dtype=torch.float16, device="cuda")
    st = _lib.fp8q_quantized_linear(Xd.data_ptr(), Wq.data_ptr(), s_w.data_ptr(), M, N, K, Yd.data_ptr(), 0, 0,
                                    torch.cuda.current_stream().cuda_stream)
    assert st == _lib.FP8Q_ERR_INVALID_ARG


def test_long_k_slice_falls_back_to_workspace(fq):
    # split forced to 1: 64 K blocks per CTA exceed the fused limit -> two steps
    M, N, K = 3, 512, 8192
    X = wl.random_f16((M, K), seed=3)
    W = wl.random_f16((N, K), seed=4, std=0.02)
    Wq, s_w = fq.quantize_weight_per_channel(W.cuda())
    fq.set_gemm_tuning(0, 0, 1)
    try:
        Y = fq.quantized_linear(X.cuda(), Wq, s_w, fused=True)
    finally:
        fq.set_gemm_tuning(0, 0, 0)
    assert_close_f16(to_np(Y), oracle(X, W), "long K fallback")
    assert_no_device_error()
