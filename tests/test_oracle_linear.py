"""Pins for the oracle's FP8 linear and MoE grouped linear.

'Quantized Inference for OneRec-V2' (关键证据 steps 3-4) and
'FP8量化在生成式推荐系统OneRec-V2中的优化实践' (§2.3): FP8 products, FP32 (here
FP64) accumulation, per-token x per-channel dequantization, FP16 output.

Pins:
  * exactness: when every row's amax is 448*2^j and every entry is an E4M3
    value times 2^j, quantization loses nothing and the result must equal
    fp16(X @ W^T) computed in float64 directly from the fp16 inputs, bit for bit;
  * brute force: on tiny random inputs the result stays within the analytic
    quantization error bound of the unquantized float64 product;
  * MoE: explicit per-row loops over expert groups, and the single-expert case.
"""
import numpy as np
import pytest

from oracle import e4m3_decode, e5m2_decode, linear_f64_unquantized, linear_ref, moe_ref, quant_rows, quant_tensor


FINITE_POS = e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))   # 0 .. 448


def exact_matrix(rng, rows, cols, j):
    """Entries = random E4M3 value * 2^j with random sign; each row holds one ±448*2^j."""
    v = rng.choice(FINITE_POS, size=(rows, cols)) * rng.choice([-1.0, 1.0], size=(rows, cols))
    where = rng.integers(0, cols, rows)
    v[np.arange(rows), where] = 448.0 * rng.choice([-1.0, 1.0], size=rows)
    m = (v * 2.0 ** j).astype(np.float16)
    assert np.all(m.astype(np.float64) == v * 2.0 ** j)     # representable in fp16
    return m


@pytest.mark.parametrize("M,N,K,jx,jw", [(7, 5, 64, -4, -6), (33, 17, 96, -2, -8), (1, 64, 256, -3, -5)])
def test_exactness_case(M, N, K, jx, jw):
    rng = np.random.default_rng(M * 1000 + N)
    X = exact_matrix(rng, M, K, jx)
    W = exact_matrix(rng, N, K, jw)
    Xq, sx = quant_rows(X)
    Wq, sw = quant_rows(W)
    assert np.all(sx == np.float32(2.0 ** jx)) and np.all(sw == np.float32(2.0 ** jw))
    Y = linear_ref(Xq, sx, Wq, sw)
    expect = (X.astype(np.float64) @ W.astype(np.float64).T).astype(np.float16)
    np.testing.assert_array_equal(Y.view(np.uint16), expect.view(np.uint16))


def quant_error_bound(X, W, sx, sw, Y):
    """Analytic bound on |Y - X W^T| for the FP8 W8A8 linear.

    Per element x: |dequant(x) - x| <= dx = max(2^-4 |x|, 2^-10 s) (3-bit
    mantissa half-ulp; subnormal half-step 2^-10 scaled by s), plus fp32
    rounding slack of the scale and product steps.  Summing products:
    |sum xhat*what - sum x*w| <= sum (|x|+dx)(|w|+dw) - |x||w|; then one
    fp16 rounding (half-ulp <= 2^-11 |y| for normals, 2^-25 below).
    """
    xa = np.abs(X.astype(np.float64))
    wa = np.abs(W.astype(np.float64))
    dx = np.maximum(2.0 ** -4 * xa, 2.0 ** -10 * sx.astype(np.float64)[:, None]) * (1 + 2.0 ** -18) + xa * 2.0 ** -20
    dw = np.maximum(2.0 ** -4 * wa, 2.0 ** -10 * sw.astype(np.float64)[:, None]) * (1 + 2.0 ** -18) + wa * 2.0 ** -20
    prod = (xa + dx) @ (wa + dw).T - xa @ wa.T
    y = np.abs(Y.astype(np.float64))
    return prod * (1 + 2.0 ** -40) + 2.0 ** -10 * y + 2.0 ** -24


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_error_bound(seed):
    rng = np.random.default_rng(100 + seed)
    M, N, K = rng.integers(1, 17, 3)
    X = (rng.standard_normal((M, K)) * np.exp(rng.uniform(-3, 3, (M, 1)))).astype(np.float16)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    Xq, sx = quant_rows(X)
    Wq, sw = quant_rows(W)
    Y = linear_ref(Xq, sx, Wq, sw)
    exact = linear_f64_unquantized(X, W)
    err = np.abs(Y.astype(np.float64) - exact)
    assert np.all(err <= quant_error_bound(X, W, sx, sw, Y))


def test_bound_is_not_vacuous():
    # The bound is tight enough to catch a transposed or dropped scale.
    rng = np.random.default_rng(1)
    X = rng.standard_normal((8, 32)).astype(np.float16)
    W = (rng.standard_normal((8, 32)) * np.linspace(0.01, 0.5, 8)[:, None]).astype(np.float16)
    Xq, sx = quant_rows(X)
    Wq, sw = quant_rows(W)
    exact = linear_f64_unquantized(X, W)
    wrong = linear_ref(Xq, sx, Wq, sw[::-1].copy())
    assert np.any(np.abs(wrong.astype(np.float64) - exact) > quant_error_bound(X, W, sx, sw, wrong))


def test_zero_rows_and_columns():
    X = np.zeros((3, 32), np.float16)
    X[1] = 1.0
    W = np.ones((4, 32), np.float16)
    W[2] = 0
    Xq, sx = quant_rows(X)
    Wq, sw = quant_rows(W)
    Y = linear_ref(Xq, sx, Wq, sw).astype(np.float64)
    assert np.all(Y[0] == 0) and np.all(Y[2] == 0) and np.all(Y[:, 2] == 0)
    assert Y[1, 0] == 32.0


def _moe_loop(X, offsets, W):
    """Per-row pure restatement with unquantized float64 inputs."""
    out = np.zeros((X.shape[0], W.shape[1]))
    for e in range(W.shape[0]):
        for r in range(int(offsets[e]), int(offsets[e + 1])):
            for n in range(W.shape[1]):
                out[r, n] = float(np.dot(X[r].astype(np.float64), W[e, n].astype(np.float64)))
    return out


def test_moe_exact_groups_loop():
    rng = np.random.default_rng(4)
    E, N, K = 5, 6, 32
    counts = [3, 0, 1, 4, 0]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    X = exact_matrix(rng, R, K, -3)
    W = np.stack([exact_matrix(rng, N, K, -7) for _ in range(E)])
    Xq, sx = quant_rows(X)
    Wq, sw = quant_rows(W.reshape(E * N, K))
    Y = moe_ref(Xq, sx, offsets, Wq.reshape(E, N, K), sw.reshape(E, N))
    expect = _moe_loop(X, offsets, W).astype(np.float16)
    np.testing.assert_array_equal(Y.view(np.uint16), expect.view(np.uint16))


def test_moe_single_expert_is_linear():
    rng = np.random.default_rng(8)
    X = rng.standard_normal((20, 48)).astype(np.float16)
    W = (rng.standard_normal((12, 48)) * 0.02).astype(np.float16)
    Xq, sx = quant_rows(X)
    Wq, sw = quant_rows(W)
    Y1 = moe_ref(Xq, sx, np.array([0, 20], np.int32), Wq[None], sw[None])
    exact = linear_f64_unquantized(X, W)
    assert np.all(np.abs(Y1.astype(np.float64) - exact) <= quant_error_bound(X, W, sx, sw, Y1))


def test_moe_rejects_bad_offsets():
    Xq = np.zeros((4, 16), np.uint8)
    sx = np.ones(4, np.float32)
    Wq = np.zeros((2, 8, 16), np.uint8)
    sw = np.ones((2, 8), np.float32)
    for bad in ([0, 3, 2], [1, 2, 4], [0, 2, 5]):
        with pytest.raises(ValueError):
            moe_ref(Xq, sx, np.array(bad, np.int32), Wq, sw)


# ---------------------------------------------------------------------------
# E5M2 activations ('FP8量化在生成式推荐系统OneRec-V2中的优化实践' §2.2).

E5M2_POS = e5m2_decode(np.arange(0, 0x7C, dtype=np.uint8))    # 0 .. 57344


def exact_matrix_e5m2(rng, rows, cols, j):
    """Entries = random E5M2 value * 2^j; each row holds one ±57344*2^j (fp16-exact for j <= 0)."""
    v = rng.choice(E5M2_POS[E5M2_POS <= 57344.0], size=(rows, cols)) * rng.choice([-1.0, 1.0], size=(rows, cols))
    v = np.where(np.abs(v) * 2.0 ** j < 2.0 ** -14, 0.0, v)            # fp16 normals hold every E5M2 value exactly
    where = rng.integers(0, cols, rows)
    v[np.arange(rows), where] = 57344.0 * rng.choice([-1.0, 1.0], size=rows)
    m = (v * 2.0 ** j).astype(np.float16)
    assert np.all(m.astype(np.float64) == v * 2.0 ** j)
    return m


@pytest.mark.parametrize("M,N,K,jx,jw", [(5, 7, 64, -12, -6), (19, 9, 128, -10, -8)])
def test_e5m2_exactness_case(M, N, K, jx, jw):
    rng = np.random.default_rng(M * 77 + N)
    X = exact_matrix_e5m2(rng, M, K, jx)
    W = exact_matrix(rng, N, K, jw)
    Xq, sx = quant_rows(X, "e5m2")
    Wq, sw = quant_rows(W)
    assert np.all(sx == np.float32(2.0 ** jx))
    Y = linear_ref(Xq, sx, Wq, sw, x_fmt="e5m2")
    expect = (X.astype(np.float64) @ W.astype(np.float64).T).astype(np.float16)
    np.testing.assert_array_equal(Y.view(np.uint16), expect.view(np.uint16))


def quant_error_bound_e5m2(X, W, sx, sw, Y):
    """As quant_error_bound, with the activation term of a 2-bit mantissa:
    dx = max(2^-3 |x|, 2^-17 s) (E5M2 half-ulp; subnormal half-step 2^-17)."""
    xa = np.abs(X.astype(np.float64))
    wa = np.abs(W.astype(np.float64))
    dx = np.maximum(2.0 ** -3 * xa, 2.0 ** -17 * sx.astype(np.float64)[:, None]) * (1 + 2.0 ** -18) + xa * 2.0 ** -20
    dw = np.maximum(2.0 ** -4 * wa, 2.0 ** -10 * sw.astype(np.float64)[:, None]) * (1 + 2.0 ** -18) + wa * 2.0 ** -20
    prod = (xa + dx) @ (wa + dw).T - xa @ wa.T
    y = np.abs(Y.astype(np.float64))
    return prod * (1 + 2.0 ** -40) + 2.0 ** -10 * y + 2.0 ** -24


@pytest.mark.parametrize("seed", range(4))
def test_e5m2_brute_force_error_bound(seed):
    rng = np.random.default_rng(300 + seed)
    M, N, K = rng.integers(1, 17, 3)
    X = (rng.standard_normal((M, K)) * np.exp(rng.uniform(-3, 3, (M, 1)))).astype(np.float16)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    Xq, sx = quant_rows(X, "e5m2")
    Wq, sw = quant_rows(W)
    Y = linear_ref(Xq, sx, Wq, sw, x_fmt="e5m2")
    err = np.abs(Y.astype(np.float64) - linear_f64_unquantized(X, W))
    assert np.all(err <= quant_error_bound_e5m2(X, W, sx, sw, Y))
    # decoding the E5M2 codes as E4M3 would be wrong: the bound must catch it
    wrong = linear_ref(Xq, sx, Wq, sw)
    finite = np.isfinite(wrong.astype(np.float64))
    assert np.any(~finite) or np.any(np.abs(wrong.astype(np.float64) - linear_f64_unquantized(X, W))
                                     > quant_error_bound_e5m2(X, W, sx, sw, wrong))


def test_per_tensor_weights_linear_error_bound():
    rng = np.random.default_rng(51)
    X = rng.standard_normal((9, 64)).astype(np.float16)
    W = (rng.standard_normal((12, 64)) * np.linspace(0.005, 0.1, 12)[:, None]).astype(np.float16)
    Xq, sx = quant_rows(X)
    Wq, sw = quant_tensor(W)
    Y = linear_ref(Xq, sx, Wq, sw)
    err = np.abs(Y.astype(np.float64) - linear_f64_unquantized(X, W))
    assert np.all(err <= quant_error_bound(X, W, sx, sw, Y))


# ---------------------------------------------------------------------------
# Row gather of the MoE grouped linear (tokens quantized once, rows read by index).

def test_per_row_quantization_commutes_with_row_gather():
    rng = np.random.default_rng(61)
    X = (rng.standard_normal((40, 96)) * np.exp(rng.uniform(-3, 3, (40, 1)))).astype(np.float16)
    idx = rng.integers(0, 40, size=70)                 # repeats, like top-2 routing
    q_all, s_all = quant_rows(X)
    q_sel, s_sel = quant_rows(X[idx])
    np.testing.assert_array_equal(q_all[idx], q_sel)
    np.testing.assert_array_equal(s_all[idx].view(np.uint32), s_sel.view(np.uint32))


def test_moe_gather_matches_permuted_rows_and_identity():
    from fp8_quantized_generative_b200 import workloads as wl
    from oracle import moe_gather_ref
    rng = np.random.default_rng(63)
    T, E, N, K = 24, 4, 12, 32
    X = rng.standard_normal((T, K)).astype(np.float16)
    logits = rng.standard_normal((T, E)).astype(np.float16)
    experts = wl.route_top2(logits)
    row_token, offsets = wl.group_by_expert(experts, E)
    W = (rng.standard_normal((E, N, K)) * 0.05).astype(np.float16)
    q = [quant_rows(W[e]) for e in range(E)]
    Wq = np.stack([c for c, _ in q]); sw = np.stack([s for _, s in q])
    xq, sx = quant_rows(X)
    xq_p, sx_p = quant_rows(X[row_token])
    got = moe_gather_ref(xq, sx, row_token, offsets, Wq, sw)
    np.testing.assert_array_equal(got.view(np.uint16), moe_ref(xq_p, sx_p, offsets, Wq, sw).view(np.uint16))
    # identity gather on already grouped rows
    ident = np.arange(len(row_token))
    np.testing.assert_array_equal(moe_gather_ref(xq_p, sx_p, ident, offsets, Wq, sw).view(np.uint16),
                                  moe_ref(xq_p, sx_p, offsets, Wq, sw).view(np.uint16))
    with pytest.raises(ValueError):
        moe_gather_ref(xq, sx, np.array([0, T]), np.array([0, 2]), Wq[:1], sw[:1])


# ---------------------------------------------------------------------------
# Top-k combine in the down projection's epilogue (FP16 scatter-add).

def _moe_setup(seed, T=30, E=5, N=16, K=48):
    from fp8_quantized_generative_b200 import workloads as wl
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, E)).astype(np.float16)
    experts = wl.route_top2(logits)
    row_token, offsets = wl.group_by_expert(experts, E)
    row_w = wl.row_weights(wl.gate_weights(logits, experts), experts)
    H = rng.standard_normal((len(row_token), K)).astype(np.float16)
    W = (rng.standard_normal((E, N, K)) * 0.05).astype(np.float16)
    hq, sh = quant_rows(H)
    q = [quant_rows(W[e]) for e in range(E)]
    Wq = np.stack([c for c, _ in q]); sw = np.stack([s for _, s in q])
    return T, row_token, offsets, row_w, hq, sh, Wq, sw


def test_combine_with_one_hot_weights_returns_the_rows():
    from oracle import moe_combine_ref
    T, row_token, offsets, _, hq, sh, Wq, sw = _moe_setup(71)
    # weight 1 on each token's first row, 0 on the other: the output is that row of moe_ref
    first = np.zeros(len(row_token), np.float32)
    seen = set()
    for r in np.argsort(row_token, kind="stable"):
        if row_token[r] not in seen:
            first[r] = 1.0
            seen.add(row_token[r])
    out = moe_combine_ref(hq, sh, offsets, Wq, sw, row_token, first, T)
    Y = moe_ref(hq, sh, offsets, Wq, sw)
    for r in np.nonzero(first)[0]:
        np.testing.assert_array_equal(out[row_token[r]].view(np.uint16), Y[r].view(np.uint16))


def test_combine_matches_an_explicit_per_token_loop():
    from oracle import moe_combine_ref
    T, row_token, offsets, row_w, hq, sh, Wq, sw = _moe_setup(73)
    out = moe_combine_ref(hq, sh, offsets, Wq, sw, row_token, row_w, T)
    # restatement: y of every row from unquantized-arithmetic building blocks, then per token
    E = Wq.shape[0]
    expert_of = np.searchsorted(offsets.astype(np.int64), np.arange(len(row_token)), side="right") - 1
    for t in range(T):
        rows = np.nonzero(row_token == t)[0]
        assert len(rows) == 2
        acc = np.float16(0.0)
        for r in rows:
            e = expert_of[r]
            yv = (e4m3_decode(hq[r])[None, :] @ e4m3_decode(Wq[e]).T)[0] * np.float64(sh[r]) * sw[e].astype(np.float64)
            c = (np.float64(row_w[r]) * yv).astype(np.float16)
            acc = (np.asarray(acc, np.float64) + c.astype(np.float64)).astype(np.float16)
        np.testing.assert_array_equal(out[t].view(np.uint16), np.asarray(acc).view(np.uint16))


def test_combine_is_within_fp16_rounding_of_the_weighted_sum():
    from oracle import moe_combine_ref
    T, row_token, offsets, row_w, hq, sh, Wq, sw = _moe_setup(79, T=64, E=6, N=32, K=64)
    out = moe_combine_ref(hq, sh, offsets, Wq, sw, row_token, row_w, T).astype(np.float64)
    Y = moe_ref(hq, sh, offsets, Wq, sw)   # fp16 rows
    exact = np.zeros_like(out)
    mag = np.zeros_like(out)
    np.add.at(exact, row_token, row_w[:, None].astype(np.float64) * Y.astype(np.float64))
    np.add.at(mag, row_token, np.abs(row_w[:, None].astype(np.float64) * Y.astype(np.float64)))
    # three fp16 roundings (each row's y, each contribution, the sum): <= 2^-10 of the magnitudes
    assert np.all(np.abs(out - exact) <= 2.0 ** -10 * (mag + np.abs(exact)) + 2.0 ** -24)


def test_combine_hand_worked_fixture():
    """tests/golden/moe_combine_hand.json: values derived by hand (exact in fp16)."""
    import json
    import os
    from oracle import moe_combine_ref
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "moe_combine_hand.json")))
    R, K = len(g["row_token"]), g["K"]
    Xq = np.zeros((R, K), np.uint8)
    Xq[:, 0] = g["x_code_k0"]
    Wq = np.zeros((g["E"], g["N"], K), np.uint8)
    Wq[:, :, 0] = g["w_code_k0"]
    out = moe_combine_ref(Xq, np.array(g["s_x"], np.float32), np.array(g["offsets"]), Wq,
                          np.array(g["s_w"], np.float32), np.array(g["row_token"]),
                          np.array(g["row_weight"], np.float32), g["tokens"])
    assert out.dtype == np.float16
    np.testing.assert_array_equal(out.astype(np.float64), np.array(g["expected"], np.float64))
