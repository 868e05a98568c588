"""GPU parity of the one-kernel quantize + FP8 linear + dequantize for M > 128
(fp8q_quantized_linear_overlapped; 'FP8量化在生成式推荐系统OneRec-V2中的优化实践'
§2.3, the QuantizeLinear + GEMM + Dequantize fusion): the CTA-pair GEMM's own
warps quantize the fp16 rows while its tensor cores start on the row blocks
already published.

* the codes and scales it leaves in the workspace are bit-exact against
  oracle.quant_rows (every row, the full QKV size included);
* Y is within the path's tolerance of oracle.linear_ref, and bitwise equal to
  the two-launch path (same tiles, same accumulation order);
* the sync words are zero again after every call, so calls repeat (with the
  same or a smaller M) and give the same bits.
"""
import numpy as np
import pytest
import torch

from oracle import linear_ref, quant_rows
from fp8_quantized_generative_b200 import workloads as wl

from parity import Guards, assert_close_f16, assert_no_device_error, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import fp8_quantized_generative_b200 as m
    assert torch.cuda.is_available()
    return m


def run(fq, X, W, ws=None):
    Wq, s_w = fq.quantize_weight_per_channel(W.cuda())
    Xd = X.cuda()
    M, K = X.shape
    g = Guards()
    if ws is None:
        # guard-banded workspace: codes, scales and sync words
        ws = (g((M, K), torch.uint8, 0xFF, "Xq_ws"), g((M,), torch.float32, float("nan"), "s_x_ws"),
              g((int(fq._lib.fp8q_overlap_sync_words(M)),), torch.int32, 0, "sync"))
    Y = g((M, W.shape[0]), torch.float16, float("nan"), "Y")
    fq.quantized_linear_overlapped(Xd, Wq, s_w, workspace=ws, out=Y)
    g.check(f"overlapped {M}x{W.shape[0]}x{K}")
    return Y, ws, (Xd, Wq, s_w)


@pytest.mark.parametrize("M,N,K", [(129, 264, 272), (300, 520, 384), (1000, 1024, 2048), (777, 512, 4096),
                                   (2048, 384, 128)])
def test_against_oracle_and_two_step(fq, M, N, K):
    X = wl.random_f16((M, K), seed=M + K, std=2.0)
    X[M // 2, 3] = 900.0                                  # one outlier row
    W = wl.random_f16((N, K), seed=N + 1, std=0.02)
    Y, (Xq, s_x, sync), (Xd, Wq, s_w) = run(fq, X, W)
    ref_q, ref_s = quant_rows(X.numpy())
    assert np.array_equal(to_np(Xq), ref_q)
    assert np.array_equal(to_np(s_x).view(np.uint32), ref_s.view(np.uint32))
    rwq, rsw = quant_rows(W.numpy())
    assert_close_f16(to_np(Y), linear_ref(ref_q, ref_s, rwq, rsw), f"overlapped {M}x{N}x{K}")
    assert torch.all(sync == 0)
    Y2 = fq.quantized_linear(Xd, Wq, s_w)
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    assert_no_device_error()


def test_repeated_calls_and_smaller_m_reuse_the_workspace(fq):
    K, N = 1024, 768
    big = fq.overlap_workspace(1500, K, "cuda")
    W = wl.random_f16((N, K), seed=5, std=0.02)
    X = wl.random_f16((1500, K), seed=6)
    first, _, _ = run(fq, X, W, ws=big)
    for _ in range(4):
        again, _, _ = run(fq, X, W, ws=big)
        assert torch.equal(first.view(torch.int16), again.view(torch.int16))
    # a smaller M on the same buffers (views of the first rows)
    X2 = wl.random_f16((600, K), seed=7)
    ws2 = (big[0][:600], big[1][:600], big[2])
    Y2, _, (Xd, Wq, s_w) = run(fq, X2, W, ws=ws2)
    ref = fq.quantized_linear(Xd, Wq, s_w)
    torch.cuda.synchronize()
    assert torch.equal(Y2.view(torch.int16), ref.view(torch.int16))
    assert torch.all(big[2] == 0)
    assert_no_device_error()


def test_small_m_runs_the_two_step_path(fq):
    M, N, K = 64, 256, 512
    X = wl.random_f16((M, K), seed=8)
    W = wl.random_f16((N, K), seed=9, std=0.02)
    Y, (Xq, s_x, sync), _ = run(fq, X, W)
    ref_q, ref_s = quant_rows(X.numpy())
    rwq, rsw = quant_rows(W.numpy())
    assert_close_f16(to_np(Y), linear_ref(ref_q, ref_s, rwq, rsw), "overlapped small M")
    assert np.array_equal(to_np(Xq), ref_q)
    assert torch.all(sync == 0)


@pytest.mark.parametrize("bn", [128, 192, 256])
def test_tile_widths(fq, bn):
    fq.set_gemm_tuning(0, bn, 0)
    try:
        M, N, K = 700, 1152, 512
        X = wl.random_f16((M, K), seed=bn)
        W = wl.random_f16((N, K), seed=bn + 1, std=0.02)
        Y, (Xq, s_x, _), _ = run(fq, X, W)
        ref_q, ref_s = quant_rows(X.numpy())
        rwq, rsw = quant_rows(W.numpy())
        assert_close_f16(to_np(Y), linear_ref(ref_q, ref_s, rwq, rsw), f"overlapped bn={bn}")
        assert_no_device_error()
    finally:
        fq.set_gemm_tuning(0, 0, 0)


def test_qkv_projection(fq):
    # the full QKV projection: every code, scale and output element
    lin = wl.qkv()
    Y, (Xq, s_x, _), _ = run(fq, lin.X, lin.W)
    ref_q, ref_s = quant_rows(lin.X.numpy())
    assert np.array_equal(to_np(Xq), ref_q)
    assert np.array_equal(to_np(s_x).view(np.uint32), ref_s.view(np.uint32))
    rwq, rsw = quant_rows(lin.W.numpy())
    assert_close_f16(to_np(Y), linear_ref(ref_q, ref_s, rwq, rsw), "overlapped qkv")
    assert_no_device_error()
