"""GPU parity of the MoE grouped linear that reads its rows from the token
matrix (fp8q_moe_grouped_linear_gather): tokens quantized once, row r of the
grouped product reads token row_token[r] (the FP16 top-2 router's grouping).
Outputs within the path's tolerance of oracle.moe_gather_ref, and equal to
the grouped linear on a gathered copy.
"""
import numpy as np
import pytest
import torch

from oracle import moe_gather_ref, quant_rows
from fp8_quantized_generative_b200 import workloads as wl

from parity import Guards, assert_close_f16, assert_no_device_error, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import fp8_quantized_generative_b200 as m
    assert torch.cuda.is_available()
    return m


def routed(T, E, seed):
    logits = wl.random_f16((T, E), seed=seed).numpy()
    row_token, offsets = wl.group_by_expert(wl.route_top2(logits), E)
    return row_token.astype(np.int32), np.asarray(offsets, dtype=np.int32)


def run_gather(fq, X, row_token, offsets, W):
    Xq, s_x = fq.quantize_rows_dynamic(X.cuda())
    Wq, s_w = fq.quantize_weight_per_channel(W.cuda())
    g = Guards()
    Y = g((len(row_token), W.shape[1]), torch.float16, float("nan"), "Y")
    fq.moe_grouped_linear_gather(Xq, s_x, torch.from_numpy(row_token).cuda(), torch.from_numpy(offsets).cuda(),
                                 Wq, s_w, out=Y)
    g.check("gather")
    return Y, (Xq, s_x, Wq, s_w)


def oracle_gather(X, row_token, offsets, W, rows=None):
    E, N, K = W.shape
    xq, sx = quant_rows(X.numpy())
    q = [quant_rows(W[e].numpy()) for e in range(E)]
    Wq = np.stack([c for c, _ in q])
    sw = np.stack([s for _, s in q])
    ref = moe_gather_ref(xq, sx, row_token, offsets, Wq, sw)
    return ref if rows is None else ref[rows]


@pytest.mark.parametrize("T,E,N,K", [(40, 6, 264, 272), (300, 8, 256, 512), (1, 3, 64, 128)])
def test_routed_small(fq, T, E, N, K):
    row_token, offsets = routed(T, E, seed=T + E)
    X = wl.random_f16((T, K), seed=T * 3 + 1)
    W = wl.random_f16((E, N, K), seed=E * 5 + 2, std=0.02)
    Y, _ = run_gather(fq, X, row_token, offsets, W)
    assert_close_f16(to_np(Y), oracle_gather(X, row_token, offsets, W), f"gather T={T} E={E}")
    assert_no_device_error()


def test_equals_grouped_linear_on_gathered_copy(fq):
    T, E, N, K = 500, 10, 512, 1024
    row_token, offsets = routed(T, E, seed=9)
    X = wl.random_f16((T, K), seed=10)
    W = wl.random_f16((E, N, K), seed=11, std=0.02)
    Y, (Xq, s_x, Wq, s_w) = run_gather(fq, X, row_token, offsets, W)
    idx = torch.from_numpy(row_token.astype(np.int64)).cuda()
    Y2 = fq.moe_grouped_linear(Xq[idx].contiguous(), s_x[idx].contiguous(), torch.from_numpy(offsets).cuda(), Wq, s_w)
    torch.cuda.synchronize()
    # same codes, scales, tiles and accumulation order: bitwise equal
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))


def test_bad_token_index_is_reported(fq):
    T, E, N, K = 8, 2, 64, 128
    X = wl.random_f16((T, K), seed=3).cuda()
    Xq, s_x = fq.quantize_rows_dynamic(X)
    Wq, s_w = fq.quantize_weight_per_channel(wl.random_f16((E, N, K), seed=4, std=0.02).cuda())
    row_token = torch.tensor([0, 1, 2, 9, 4, 5], dtype=torch.int32, device="cuda")      # 9 >= T
    offsets = torch.tensor([0, 3, 6], dtype=torch.int32, device="cuda")
    fq.moe_grouped_linear_gather(Xq, s_x, row_token, offsets, Wq, s_w)
    assert fq.device_error() == 0x8


def test_moe_up_from_tokens(fq):
    # every grouped row of the full-size up projection read from the token matrix
    m = wl.moe()
    row_token = np.asarray(m.token_of_row, dtype=np.int32)
    offsets = np.asarray(m.offsets, dtype=np.int32)
    Y, _ = run_gather(fq, m.X, row_token, offsets, m.W_up)
    assert_close_f16(to_np(Y), oracle_gather(m.X, row_token, offsets, m.W_up), "moe up from tokens")
    assert_no_device_error()


# ------------------------------------------------- dispatch in the quantizer's store

def run_dispatch(fq, X, token_rows, R, fmt="e4m3"):
    # guard-banded outputs: a token row dispatched past the last grouped row
    # (or a scale written past the scale array) changes the guard bytes
    g = Guards()
    Xq = g((R, X.shape[1]), torch.uint8, 0x7F, "Xq")
    s = g((R,), torch.float32, float("nan"), "s_x")
    fq.quantize_rows_dispatch(X.cuda(), torch.from_numpy(token_rows).cuda(), R, out=(Xq, s), fmt=fmt)
    g.check("dispatch")
    return to_np(Xq), to_np(s)


@pytest.mark.parametrize("T,E,K", [(40, 6, 272), (300, 8, 2048), (5, 3, 16), (9, 4, 20480)])
@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_dispatch_bit_exact(fq, T, E, K, fmt):
    # grouped row r holds the codes and scale of token row_token[r] (K = 20480: the two-pass kernel)
    row_token, _ = routed(T, E, seed=T + K)
    R = len(row_token)
    X = wl.random_f16((T, K), seed=K + 1, std=2.0)
    got_q, got_s = run_dispatch(fq, X, wl.token_rows(row_token, T), R, fmt)
    ref_q, ref_s = quant_rows(X.numpy(), fmt)
    assert np.array_equal(got_q, ref_q[row_token])
    assert np.array_equal(got_s.view(np.uint32), ref_s[row_token].view(np.uint32))
    assert_no_device_error()


def test_dispatch_skips_minus_one_and_reports_bad_rows(fq):
    T, K, R = 4, 128, 5
    X = wl.random_f16((T, K), seed=2)
    tr = np.array([[0, 3], [-1, -1], [1, -1], [4, 2]], np.int32)
    got_q, got_s = run_dispatch(fq, X, tr, R)
    ref_q, ref_s = quant_rows(X.numpy())
    for t, r in [(0, 0), (0, 3), (2, 1), (3, 4), (3, 2)]:
        assert np.array_equal(got_q[r], ref_q[t]) and got_s[r] == ref_s[t]
    assert_no_device_error()
    bad = np.array([[0, 5], [1, -2], [2, -1], [3, -1]], np.int32)     # 5 >= R, -2 < -1
    got_q, _ = run_dispatch(fq, X, bad, R)
    assert fq.device_error() == 0x8
    assert np.array_equal(got_q[0], ref_q[0]) and np.all(got_q[4] == 0x7F)


def test_dispatch_then_grouped_linear_equals_gather(fq):
    # quantize once and scatter, then the plain grouped linear: bitwise the gathered product
    T, E, N, K = 500, 10, 512, 1024
    row_token, offsets = routed(T, E, seed=9)
    X = wl.random_f16((T, K), seed=10)
    W = wl.random_f16((E, N, K), seed=11, std=0.02)
    Y, (_, _, Wq, s_w) = run_gather(fq, X, row_token, offsets, W)
    Xq_g, s_g = fq.quantize_rows_dispatch(X.cuda(), torch.from_numpy(wl.token_rows(row_token, T)).cuda(),
                                          len(row_token))
    fq.set_gemm_tuning(1, 0, 0)
    try:
        Y2 = fq.moe_grouped_linear(Xq_g, s_g, torch.from_numpy(offsets).cuda(), Wq, s_w)
        torch.cuda.synchronize()
    finally:
        fq.set_gemm_tuning(0, 0, 0)
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))


def test_dispatch_moe_tokens(fq):
    # every grouped row of the full-size dispatch, bit for bit
    m = wl.moe()
    row_token = np.asarray(m.token_of_row, dtype=np.int32)
    T = m.X.shape[0]
    got_q, got_s = run_dispatch(fq, m.X, wl.token_rows(row_token, T), len(row_token))
    ref_q, ref_s = quant_rows(m.X.numpy())
    assert np.array_equal(got_q, ref_q[row_token])
    assert np.array_equal(got_s.view(np.uint32), ref_s[row_token].view(np.uint32))
    assert_no_device_error()
