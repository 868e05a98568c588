"""GPU parity of the MoE down projection with the top-2 combine in its
epilogue (fp8q_moe_grouped_linear_combine; 'FP8量化在生成式推荐系统OneRec-V2中的
优化实践' §3.2 and the OneRec-V2 item on per-token/expert-aligned quantization
of the MoE layer): grouped row r adds fp16(row_weight[r] * y[r]) into output
row row_token[r] with an FP16 atomic add.

Tolerance.  out[t] = c1 + c2 can cancel, so an error bound relative to
|out[t]| is wrong; each contribution carries the grouped linear's error
(2^-9 |c| + 1e-3 rms) and the sum one more fp16 rounding on either side, so
the bound is taken against S[t] = sum_r |row_weight[r] * y[r]|:
    per element:  |out_gpu - out_ref| <= 2^-9 * (S + |out_ref|) + 1e-3 * rms(S)
    whole tensor: ||out_gpu - out_ref||_F <= 1e-3 * ||S||_F
Every token row of the full-size combine is compared, with guard-banded
outputs, and the whole MoE layer (dispatch, up, re-quantize, down + combine)
is checked stage by stage at full size.
Kernel-against-kernel checks are bitwise: with unit weights the combine
equals the fp16 scatter-add (one rounding of the exact sum) of the plain
grouped linear's outputs, since the same tiles produce the same fp32 values.
"""
import numpy as np
import pytest
import torch

from oracle import moe_combine_ref, moe_ref, quant_rows
from fp8_quantized_generative_b200 import workloads as wl

from parity import Guards, assert_close_f16, assert_no_device_error, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import fp8_quantized_generative_b200 as m
    assert torch.cuda.is_available()
    return m


def routed(T, E, seed, topk=2):
    logits = wl.random_f16((T, E), seed=seed).numpy()
    experts = wl.route_top2(logits, topk=topk)
    row_token, offsets = wl.group_by_expert(experts, E)
    w = wl.row_weights(wl.gate_weights(logits, experts), experts)
    return row_token.astype(np.int32), np.asarray(offsets, dtype=np.int32), w.astype(np.float32)


def oracle_quant(X, W):
    E, N, K = W.shape
    xq, sx = quant_rows(X.numpy())
    q = [quant_rows(W[e].numpy()) for e in range(E)]
    return xq, sx, np.stack([c for c, _ in q]), np.stack([s for _, s in q])


def assert_close_combine(got, ref, S, what):
    g = np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape and np.all(np.isfinite(g)), what
    rms = float(np.sqrt(np.mean(S * S)))
    bound = 2.0 ** -9 * (S + np.abs(r)) + 1e-3 * rms
    bad = np.abs(g - r) > bound
    if np.any(bad):
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {int(bad.sum())} out of tolerance; first at {i}: gpu={g[i]!r} "
                             f"ref={r[i]!r} bound={bound[i]!r}")
    assert np.linalg.norm(g - r) <= 1e-3 * np.linalg.norm(S), what


def magnitude_sum(xq, sx, offsets, wq, sw, row_token, w, T):
    """S[t] = sum over t's rows of |w_r * y_r| (y from the oracle's grouped linear)."""
    y = moe_ref(xq, sx, offsets, wq, sw).astype(np.float64)
    S = np.zeros((T, y.shape[1]))
    np.add.at(S, row_token.astype(np.int64), np.abs(w.astype(np.float64))[:, None] * np.abs(y))
    return S


def run_combine(fq, Xp, offsets, W, row_token, w, T):
    g = Guards()
    E, N, K = W.shape
    R = Xp.shape[0]
    Xq = g((R, K), torch.uint8, 0xFF, "Xq")
    s_x = g((R,), torch.float32, float("nan"), "s_x")
    fq.quantize_rows_dynamic(Xp.cuda(), out=(Xq, s_x))
    Wq = g((E, N, K), torch.uint8, 0xFF, "Wq")
    s_w = g((E, N), torch.float32, float("nan"), "s_w")
    fq.quantize_weight_per_channel(W.cuda(), out=(Wq, s_w))
    # guard-banded output: an atomic add into a token row past the end (or a
    # clear that runs over) changes the guard bytes
    out = g((T, N), torch.float16, float("nan"), "out")
    fq.moe_grouped_linear_combine(Xq, s_x, torch.from_numpy(offsets).cuda(), Wq, s_w,
                                  torch.from_numpy(row_token).cuda(), torch.from_numpy(w).cuda(), T, out=out)
    g.check(f"combine T={T} E={E} N={N} K={K}")
    return out, (Xq, s_x, Wq, s_w)


@pytest.mark.parametrize("T,E,N,K", [(40, 6, 264, 272), (300, 8, 256, 512), (1, 3, 64, 128), (700, 5, 136, 1040)])
def test_routed_top2_against_oracle(fq, T, E, N, K):
    row_token, offsets, w = routed(T, E, seed=T + 7 * E)
    Xp = wl.random_f16((len(row_token), K), seed=T + K)
    W = wl.random_f16((E, N, K), seed=E + N, std=0.02)
    out, _ = run_combine(fq, Xp, offsets, W, row_token, w, T)
    xq, sx, wq, sw = oracle_quant(Xp, W)
    ref = moe_combine_ref(xq, sx, offsets, wq, sw, row_token, w, T)
    S = magnitude_sum(xq, sx, offsets, wq, sw, row_token, w, T)
    assert_close_combine(to_np(out), ref, S, f"combine T={T} E={E} N={N} K={K}")
    assert_no_device_error()


def test_tokens_without_rows_are_zero(fq):
    T, E, N, K = 50, 3, 128, 256
    row_token = np.array([0, 3, 3, 7, 0, 9], np.int32)        # tokens 1,2,4,5,6,8,10.. get nothing
    offsets = np.array([0, 2, 2, 6], np.int32)
    w = np.array([0.25, 0.5, 0.5, 1.0, 0.75, -0.5], np.float32)
    Xp = wl.random_f16((6, K), seed=5)
    W = wl.random_f16((E, N, K), seed=6, std=0.02)
    out, _ = run_combine(fq, Xp, offsets, W, row_token, w, T)
    xq, sx, wq, sw = oracle_quant(Xp, W)
    ref = moe_combine_ref(xq, sx, offsets, wq, sw, row_token, w, T)
    S = magnitude_sum(xq, sx, offsets, wq, sw, row_token, w, T)
    assert_close_combine(to_np(out), ref, S, "sparse tokens")
    untouched = np.setdiff1d(np.arange(T), row_token)
    assert np.all(to_np(out)[untouched].view(np.uint16) == 0)        # +0.0 exactly
    assert_no_device_error()


def test_no_rows_clears_output(fq):
    T, E, N, K = 9, 2, 64, 128
    out = torch.full((T, N), 3.0, dtype=torch.float16, device="cuda")
    Xq = torch.empty((0, K), dtype=torch.uint8, device="cuda")
    s_x = torch.empty((0,), dtype=torch.float32, device="cuda")
    Wq, s_w = fq.quantize_weight_per_channel(wl.random_f16((E, N, K), seed=1, std=0.02).cuda())
    off = torch.zeros(E + 1, dtype=torch.int32, device="cuda")
    e32 = torch.empty((0,), dtype=torch.int32, device="cuda")
    ef = torch.empty((0,), dtype=torch.float32, device="cuda")
    fq.moe_grouped_linear_combine(Xq, s_x, off, Wq, s_w, e32, ef, T, out=out)
    torch.cuda.synchronize()
    assert torch.all(out == 0)


@pytest.mark.parametrize("topk", [1, 2])
def test_unit_weights_equal_scatter_add_of_grouped_linear(fq, topk):
    T, E, N, K = 400, 7, 512, 768
    row_token, offsets, _ = routed(T, E, seed=21 + topk, topk=topk)
    ones = np.ones(len(row_token), np.float32)
    Xp = wl.random_f16((len(row_token), K), seed=22)
    W = wl.random_f16((E, N, K), seed=23, std=0.02)
    out, (Xq, s_x, Wq, s_w) = run_combine(fq, Xp, offsets, W, row_token, ones, T)
    fq.set_gemm_tuning(1, 0, 0)           # the single-CTA grouped kernel, as the combine uses
    try:
        Y = fq.moe_grouped_linear(Xq, s_x, torch.from_numpy(offsets).cuda(), Wq, s_w)
        torch.cuda.synchronize()
    finally:
        fq.set_gemm_tuning(0, 0, 0)
    y = to_np(Y).astype(np.float64)
    exp = np.zeros((T, N), np.float64)
    np.add.at(exp, row_token.astype(np.int64), y)          # exact: two fp16 values sum exactly in fp64
    exp = exp.astype(np.float16)
    assert np.array_equal(to_np(out).view(np.uint16), exp.view(np.uint16))


def test_repeatable_bitwise(fq):
    T, E, N, K = 600, 8, 384, 512
    row_token, offsets, w = routed(T, E, seed=31)
    Xp = wl.random_f16((len(row_token), K), seed=32)
    W = wl.random_f16((E, N, K), seed=33, std=0.02)
    a, _ = run_combine(fq, Xp, offsets, W, row_token, w, T)
    b, _ = run_combine(fq, Xp, offsets, W, row_token, w, T)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_bad_token_is_reported(fq):
    T, E, N, K = 8, 2, 64, 128
    Xq, s_x = fq.quantize_rows_dynamic(wl.random_f16((6, K), seed=3).cuda())
    Wq, s_w = fq.quantize_weight_per_channel(wl.random_f16((E, N, K), seed=4, std=0.02).cuda())
    row_token = torch.tensor([0, 1, 2, 8, 4, 5], dtype=torch.int32, device="cuda")      # 8 >= T
    w = torch.ones(6, dtype=torch.float32, device="cuda")
    offsets = torch.tensor([0, 3, 6], dtype=torch.int32, device="cuda")
    fq.moe_grouped_linear_combine(Xq, s_x, offsets, Wq, s_w, row_token, w, T)
    assert fq.device_error() == 0x8


def test_moe_down_combine(fq):
    # every token row of the full-size down projection + combine
    m = wl.moe()
    row_token = np.asarray(m.token_of_row, dtype=np.int32)
    offsets = np.asarray(m.offsets, dtype=np.int32)
    T = m.X.shape[0]
    F = wl.MOE_F
    H = wl.random_f16((len(row_token), F), seed=404)   # the expert FFN's hidden rows
    out, _ = run_combine(fq, H, offsets, m.W_down, row_token, m.row_weight, T)
    xq, sx, wq, sw = oracle_quant(H, m.W_down)
    ref = moe_combine_ref(xq, sx, offsets, wq, sw, row_token, m.row_weight, T)
    S = magnitude_sum(xq, sx, offsets, wq, sw, row_token, m.row_weight, T)
    assert_close_combine(to_np(out), ref, S, "moe down combine")
    assert_no_device_error()


def test_hand_worked_fixture_bit_exact(fq):
    # tests/golden/moe_combine_hand.json: every intermediate is exact, so the
    # GPU result must equal the hand-derived values bit for bit (channels 2..7
    # have zero weights and stay zero: the API wants N % 8 == 0)
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "moe_combine_hand.json")))
    R, K, E, N = len(g["row_token"]), g["K"], g["E"], 8
    Xq = torch.zeros((R, K), dtype=torch.uint8)
    Xq[:, 0] = torch.tensor(g["x_code_k0"], dtype=torch.uint8)
    Wq = torch.zeros((E, N, K), dtype=torch.uint8)
    Wq[:, :2, 0] = torch.tensor(g["w_code_k0"], dtype=torch.uint8)
    s_w = torch.ones((E, N), dtype=torch.float32)
    s_w[:, :2] = torch.tensor(g["s_w"], dtype=torch.float32)
    out = fq.moe_grouped_linear_combine(
        Xq.cuda(), torch.tensor(g["s_x"], dtype=torch.float32).cuda(),
        torch.tensor(g["offsets"], dtype=torch.int32).cuda(), Wq.cuda(), s_w.cuda(),
        torch.tensor(g["row_token"], dtype=torch.int32).cuda(), torch.tensor(g["row_weight"], dtype=torch.float32).cuda(),
        g["tokens"])
    torch.cuda.synchronize()
    exp = np.zeros((g["tokens"], N), np.float16)
    exp[:, :2] = np.array(g["expected"], np.float16)
    assert np.array_equal(to_np(out).view(np.uint16), exp.view(np.uint16))
    assert_no_device_error()


def test_moe_layer_chained_full(fq):
    # The whole MoE layer as the moe_tokens step runs it, at full size:
    # dispatch-quantize the 8192 tokens into their 16384 expert-grouped rows,
    # up projection, re-quantize the hidden rows, down projection with the
    # weighted top-2 combine into the token rows.  Each stage is checked
    # against the oracle on that stage's own input; the GPU's fp16 hidden
    # matrix H is an input to the oracle's re-quantization and down
    # projection (an input, not a result under test).
    m = wl.moe()
    row_token = np.asarray(m.token_of_row, dtype=np.int32)
    offsets = np.asarray(m.offsets, dtype=np.int32)
    T, D = m.X.shape
    R = len(row_token)
    E, F, _ = m.W_up.shape
    g = Guards()
    Wuq = g((E, F, D), torch.uint8, 0xFF, "Wuq")
    swu = g((E, F), torch.float32, float("nan"), "swu")
    fq.quantize_weight_per_channel(m.W_up.cuda(), out=(Wuq, swu))
    Wdq = g((E, D, F), torch.uint8, 0xFF, "Wdq")
    swd = g((E, D), torch.float32, float("nan"), "swd")
    fq.quantize_weight_per_channel(m.W_down.cuda(), out=(Wdq, swd))
    off = torch.from_numpy(offsets).cuda()
    rt = torch.from_numpy(row_token).cuda()
    Xq = g((R, D), torch.uint8, 0xFF, "Xq")
    sx = g((R,), torch.float32, float("nan"), "s_x")
    fq.quantize_rows_dispatch(m.X.cuda(), torch.from_numpy(wl.token_rows(row_token, T)).cuda(), R, out=(Xq, sx))
    H = g((R, F), torch.float16, float("nan"), "H")
    fq.moe_grouped_linear(Xq, sx, off, Wuq, swu, out=H)
    Hq = g((R, F), torch.uint8, 0xFF, "Hq")
    sh = g((R,), torch.float32, float("nan"), "s_h")
    fq.quantize_rows_dynamic(H, out=(Hq, sh))
    out = g((T, D), torch.float16, float("nan"), "out")
    fq.moe_grouped_linear_combine(Hq, sh, off, Wdq, swd, rt, torch.from_numpy(m.row_weight).cuda(), T, out=out)
    g.check("moe layer")
    assert_no_device_error()

    # dispatch: every grouped row holds its token's codes and scale, bit for bit
    tq, ts = quant_rows(m.X.numpy())
    assert np.array_equal(to_np(Xq), tq[row_token])
    assert np.array_equal(to_np(sx).view(np.uint32), ts[row_token].view(np.uint32))
    # up projection: every grouped row within the tolerance
    uq, us = oracle_quant(m.X, m.W_up)[2:]
    h = to_np(H)
    assert_close_f16(h, moe_ref(tq[row_token], ts[row_token], offsets, uq, us), "chained up")
    # re-quantization of the GPU's hidden rows, bit for bit
    hq, hs = quant_rows(h)
    assert np.array_equal(to_np(Hq), hq)
    assert np.array_equal(to_np(sh).view(np.uint32), hs.view(np.uint32))
    # down projection + combine: every token row
    dq = [quant_rows(m.W_down[e].numpy()) for e in range(E)]
    wq = np.stack([c for c, _ in dq])
    ws = np.stack([s for _, s in dq])
    ref = moe_combine_ref(hq, hs, offsets, wq, ws, row_token, m.row_weight, T)
    S = magnitude_sum(hq, hs, offsets, wq, ws, row_token, m.row_weight, T)
    assert_close_combine(to_np(out), ref, S, "chained down + combine")
