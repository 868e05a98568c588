"""GPU parity of the variants the pages describe beside the main path.

* E5M2 activations ('FP8量化在生成式推荐系统OneRec-V2中的优化实践' §2.2): the
  per-token quantizer with max_code 57344 (codes and scales bit-exact against
  oracle.quant_rows(..., "e5m2")), and the linear / MoE grouped linear with
  E5M2 x E4M3 tensor-core products (FP16 outputs within the path's tolerance
  of oracle.linear_ref(..., x_fmt="e5m2")) on every kernel family.
* Per-tensor weight scales (same page, §2.1, the FFN linears): codes and the
  replicated scale bit-exact against oracle.quant_tensor, and the linear that
  consumes them.
"""
import numpy as np
import pytest
import torch

from oracle import linear_ref, moe_ref, quant_rows, quant_tensor
from fp8_quantized_generative_b200 import workloads as wl

from parity import assert_close_f16, assert_no_device_error, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import fp8_quantized_generative_b200 as m
    assert torch.cuda.is_available()
    return m


def _assert_codes(got_q, ref_q, got_s, ref_s, what):
    if not np.array_equal(got_q, ref_q):
        bad = np.argwhere(got_q != ref_q)[0]
        raise AssertionError(f"{what}: code mismatch at {tuple(bad)}: gpu 0x{got_q[tuple(bad)]:02x} "
                             f"oracle 0x{ref_q[tuple(bad)]:02x}")
    np.testing.assert_array_equal(got_s.view(np.uint32), ref_s.view(np.uint32), err_msg=what)


def _quant_e5m2(fq, X):
    Xq = torch.full(X.shape, 0x7F, dtype=torch.uint8, device="cuda")
    s = torch.full((X.shape[0],), float("nan"), dtype=torch.float32, device="cuda")
    fq.quantize_rows_dynamic(X.cuda(), out=(Xq, s), fmt="e5m2")
    torch.cuda.synchronize()
    return Xq, s


@pytest.mark.parametrize("M,K", [(1, 16), (3, 272), (37, 1024), (129, 2064), (9, 8192), (2, 16400)])
def test_e5m2_quant_ragged_shapes(fq, M, K):
    X = wl.random_f16((M, K), seed=M * 11 + K, std=3.0)
    Xq, s = _quant_e5m2(fq, X)
    ref_q, ref_s = quant_rows(X.numpy(), "e5m2")
    _assert_codes(to_np(Xq), ref_q, to_np(s), ref_s, f"e5m2 {M}x{K}")
    assert_no_device_error()


def test_e5m2_quant_edge_rows(fq):
    K = 512
    X = wl.random_f16((6, K), seed=9).float()
    X[0] = 0.0                                   # all-zero row -> eps scale
    X[1, 7] = 60000.0                            # one huge value: the rest goes subnormal
    X[2] = X[2] * 1e-4                           # tiny row (fp16 subnormal inputs)
    X[3, ::2] = -X[3, ::2].abs()                 # mixed signs, -0.0 below
    X[4] = 0.0
    X[4, 3] = -0.0
    X[5, :] = 1.0
    X = X.half()
    Xq, s = _quant_e5m2(fq, X)
    ref_q, ref_s = quant_rows(X.numpy(), "e5m2")
    _assert_codes(to_np(Xq), ref_q, to_np(s), ref_s, "e5m2 edge rows")


def test_e5m2_quant_qkv_activations(fq):
    lin = wl.qkv()
    Xq, s = _quant_e5m2(fq, lin.X)
    ref_q, ref_s = quant_rows(lin.X.numpy(), "e5m2")
    _assert_codes(to_np(Xq), ref_q, to_np(s), ref_s, "e5m2 qkv X")


@pytest.fixture(params=[0, 1, 2, 3], ids=["auto", "single", "pair", "splitk"])
def family(request, fq):
    fq.set_gemm_tuning(request.param, 0, 0)
    yield request.param
    fq.set_gemm_tuning(0, 0, 0)


@pytest.mark.parametrize("M,N,K", [(5, 264, 272), (100, 512, 1024), (300, 520, 384)])
def test_e5m2_linear(fq, family, M, N, K):
    X = wl.random_f16((M, K), seed=M + K, std=2.0)
    W = wl.random_f16((N, K), seed=N + 3, std=0.02)
    Xq, s_x = _quant_e5m2(fq, X)
    Wq, s_w = fq.quantize_weight_per_channel(W.cuda())
    Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    fq.linear(Xq, s_x, Wq, s_w, out=Y, x_fmt="e5m2")
    torch.cuda.synchronize()
    rxq, rsx = quant_rows(X.numpy(), "e5m2")
    rwq, rsw = quant_rows(W.numpy())
    assert_close_f16(to_np(Y), linear_ref(rxq, rsx, rwq, rsw, x_fmt="e5m2"), f"e5m2 linear {M}x{N}x{K}")
    assert_no_device_error()


def test_e5m2_linear_differs_from_e4m3_reading(fq):
    # The same codes read as E4M3 give a different product: the format field reaches the MMA.
    M, N, K = 64, 256, 256
    X = wl.random_f16((M, K), seed=71, std=1.0)
    W = wl.random_f16((N, K), seed=72, std=0.02)
    Xq, s_x = _quant_e5m2(fq, X)
    Wq, s_w = fq.quantize_weight_per_channel(W.cuda())
    y5 = to_np(fq.linear(Xq, s_x, Wq, s_w, x_fmt="e5m2")).astype(np.float64)
    y4 = to_np(fq.linear(Xq, s_x, Wq, s_w)).astype(np.float64)
    torch.cuda.synchronize()
    assert np.linalg.norm(y5 - y4) > 0.1 * np.linalg.norm(y5)


@pytest.mark.parametrize("moe_family", [0, 2], ids=["single", "pair"])
def test_e5m2_moe_small_groups(fq, moe_family):
    fq.set_gemm_tuning(moe_family, 0, 0)
    try:
        E, N, K = 5, 264, 272
        counts = [0, 130, 1, 300, 57]
        off = wl.offsets_from_counts(counts)
        R = int(off[-1])
        X = wl.random_f16((R, K), seed=31)
        W = wl.random_f16((E, N, K), seed=32, std=0.02)
        Xq, s_x = _quant_e5m2(fq, X)
        Wq, s_w = fq.quantize_weight_per_channel(W.cuda())
        Y = torch.full((R, N), float("nan"), dtype=torch.float16, device="cuda")
        fq.moe_grouped_linear(Xq, s_x, torch.from_numpy(off).cuda(), Wq, s_w, out=Y, x_fmt="e5m2")
        torch.cuda.synchronize()
        rxq, rsx = quant_rows(X.numpy(), "e5m2")
        rwq, rsw = quant_rows(W.reshape(E * N, K).numpy())
        ref = moe_ref(rxq, rsx, off, rwq.reshape(E, N, K), rsw.reshape(E, N), x_fmt="e5m2")
        assert_close_f16(to_np(Y), ref, "e5m2 moe")
        assert_no_device_error()
    finally:
        fq.set_gemm_tuning(0, 0, 0)


# ---------------------------------------------------------------- per-tensor weights

@pytest.mark.parametrize("N,K", [(1, 16), (300, 272), (2048, 8192), (4096, 4096)])
def test_per_tensor_quant(fq, N, K):
    W = wl.random_f16((N, K), seed=N + K + 5, std=0.02)
    if N > 1:
        W[N // 2, K // 3] = 0.75                    # the global maximum in one row
    Wq = torch.full((N, K), 0x7F, dtype=torch.uint8, device="cuda")
    s = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
    Wq2, s2 = fq.quantize_weight_per_tensor(W.cuda())
    Wq.copy_(Wq2)
    s.copy_(s2)
    torch.cuda.synchronize()
    ref_q, ref_s = quant_tensor(W.numpy())
    _assert_codes(to_np(Wq), ref_q, to_np(s), ref_s, f"per-tensor {N}x{K}")
    assert_no_device_error()


def test_per_tensor_zero_matrix(fq):
    W = torch.zeros((64, 128), dtype=torch.float16)
    Wq, s = fq.quantize_weight_per_tensor(W.cuda())
    torch.cuda.synchronize()
    ref_q, ref_s = quant_tensor(W.numpy())
    _assert_codes(to_np(Wq), ref_q, to_np(s), ref_s, "per-tensor zeros")


def test_per_tensor_linear_ffn_up_rows(fq):
    # The FFN up shape with a per-tensor weight scale; every output row against the oracle.
    up, _ = wl.ffn()
    Wq, s_w = fq.quantize_weight_per_tensor(up.W.cuda())
    Xq, s_x = fq.quantize_rows_dynamic(up.X.cuda())
    Y = fq.linear(Xq, s_x, Wq, s_w)
    torch.cuda.synchronize()
    rxq, rsx = quant_rows(up.X.numpy())
    rwq, rsw = quant_tensor(up.W.numpy())
    assert_close_f16(to_np(Y), linear_ref(rxq, rsx, rwq, rsw), "per-tensor ffn up")
    assert_no_device_error()
