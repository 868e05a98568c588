"""Pins for the oracle's per-row quantization (per-token / per-channel scales).

Rule under test ('Quantized Inference for OneRec-V2', 关键证据 steps 1-2;
'FP8量化在生成式推荐系统OneRec-V2中的优化实践' §2.2 scale = max_code / max(|x|, eps)):
    a' = max(max|x|, 1e-12); r = fl32(448/a'); s = fl32(a'/448); q = E4M3(fl32(x*r)).
"""
import json
import os

import numpy as np
import pytest

from oracle import EPS, e4m3_decode, e5m2_decode, quant_rows, quant_tensor


def _load(golden_dir):
    with open(os.path.join(golden_dir, "quant_rows_hand.json")) as f:
        return json.load(f)["cases"]


def test_hand_worked_rows(golden_dir):
    for case in _load(golden_dir):
        x = np.array([np.float16(v) for v in case["x"]], dtype=np.float16)[None, :]
        codes, s = quant_rows(x)
        exp_codes = np.array([int(c, 16) for c in case["codes"]], dtype=np.uint8)
        np.testing.assert_array_equal(codes[0], exp_codes, err_msg=case["name"])
        assert s.dtype == np.float32
        assert int(s.view(np.uint32)[0]) == int(case["scale_f32_bits"], 16), case["name"]


def test_row_max_maps_to_448():
    # The element holding the row's amax always lands on code ±448 (0x7E/0xFE):
    # fl32(a * fl32(448/a)) is within one fp32 ulp of 448, far inside E4M3's
    # half-spacing of 16 there, and anything above 448 saturates.
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((512, 300)) * np.exp(rng.uniform(-8, 8, (512, 1)))).astype(np.float16)
    x = x.astype(np.float32)
    x = x[np.all(np.isfinite(x), axis=1) & (np.abs(x).max(axis=1) > 0)].astype(np.float16)
    codes, _ = quant_rows(x)
    idx = np.argmax(np.abs(x.astype(np.float32)), axis=1)
    picked = codes[np.arange(len(x)), idx] & 0x7F
    assert np.all(picked == 0x7E)


def test_scale_times_reciprocal_is_one_within_ulps():
    rng = np.random.default_rng(5)
    a = np.exp(rng.uniform(-20, 10, 10000)).astype(np.float16).astype(np.float32)
    a = a[a > 0]
    x = np.zeros((len(a), 2), np.float32)
    x[:, 0] = a
    _, s = quant_rows(x.astype(np.float16))
    np.testing.assert_allclose(s.astype(np.float64) * 448.0, a.astype(np.float64),
                               rtol=2 ** -23)


def test_dequant_error_bound_per_element():
    # |q*s - x| <= max(2^-4 |x|, 2^-10 s) (+ fp32 rounding slack) for every element.
    rng = np.random.default_rng(9)
    x = (rng.standard_normal((64, 512)) * np.exp(rng.uniform(-4, 4, (64, 1)))).astype(np.float16)
    x[:, 7] *= np.float16(50)
    codes, s = quant_rows(x)
    deq = e4m3_decode(codes) * s.astype(np.float64)[:, None]
    xa = np.abs(x.astype(np.float64))
    bound = np.maximum(2.0 ** -4 * xa, 2.0 ** -10 * s.astype(np.float64)[:, None]) * (1 + 2.0 ** -18) + xa * 2.0 ** -20
    assert np.all(np.abs(deq - x.astype(np.float64)) <= bound)


def test_scale_invariance_power_of_two():
    # Multiplying a row by 2^j multiplies s by 2^j and leaves the codes unchanged
    # (all steps are exact under power-of-two scaling away from the eps floor).
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((32, 128))).astype(np.float16)
    c0, s0 = quant_rows(x)
    for j in (-3, 1, 4):
        c1, s1 = quant_rows((x.astype(np.float32) * 2.0 ** j).astype(np.float16))
        np.testing.assert_array_equal(c0, c1)
        np.testing.assert_array_equal(s1, (s0 * np.float32(2.0 ** j)).astype(np.float32))


def test_sign_symmetry():
    rng = np.random.default_rng(17)
    x = rng.standard_normal((16, 64)).astype(np.float16)
    c0, s0 = quant_rows(x)
    c1, s1 = quant_rows(-x)
    np.testing.assert_array_equal(c1, c0 ^ np.uint8(0x80))
    np.testing.assert_array_equal(s0, s1)


def test_brute_force_small_rows():
    # Pure-Python restatement on a handful of values: pick the nearest E4M3
    # value by exhaustive search over all 254 finite codes, ties to the even code.
    finite = [c for c in range(256) if (c & 0x7F) != 0x7F]
    table = {c: float(e4m3_decode(np.array([c], np.uint8))[0]) for c in finite}
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((6, 40)) * 3).astype(np.float16)
    codes, s = quant_rows(x)
    for i in range(x.shape[0]):
        a = max(float(np.max(np.abs(x[i].astype(np.float32)))), float(EPS))
        r = np.float32(np.float32(448.0) / np.float32(a))
        for k in range(x.shape[1]):
            t = float(np.float32(np.float32(x[i, k]) * r))
            t = min(max(t, -448.0), 448.0)
            best = min(finite, key=lambda c: (abs(table[c] - t), c & 1,
                                              (c >> 7) != (1 if np.signbit(t) else 0)))
            assert codes[i, k] == best or (t == 0.0 and (codes[i, k] & 0x7F) == 0), (i, k, t)


def test_empty_inputs():
    c, s = quant_rows(np.zeros((0, 16), np.float16))
    assert c.shape == (0, 16) and s.shape == (0,)


# ---------------------------------------------------------------------------
# E5M2 activations ('FP8量化在生成式推荐系统OneRec-V2中的优化实践' §2.2): the same
# steps with max_code = 57344.

def test_e5m2_hand_worked_rows(golden_dir):
    with open(os.path.join(golden_dir, "quant_rows_e5m2_hand.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        x = np.array([np.float16(v) for v in case["x"]], dtype=np.float16)[None, :]
        codes, s = quant_rows(x, "e5m2")
        exp_codes = np.array([int(c, 16) for c in case["codes"]], dtype=np.uint8)
        np.testing.assert_array_equal(codes[0], exp_codes, err_msg=case["name"])
        assert int(s.view(np.uint32)[0]) == int(case["scale_f32_bits"], 16), case["name"]


def test_e5m2_row_max_maps_to_57344():
    rng = np.random.default_rng(33)
    x = (rng.standard_normal((256, 200)) * np.exp(rng.uniform(-6, 6, (256, 1)))).astype(np.float16)
    x = x[np.all(np.isfinite(x.astype(np.float32)), axis=1) & (np.abs(x.astype(np.float32)).max(axis=1) > 0)]
    codes, _ = quant_rows(x, "e5m2")
    idx = np.argmax(np.abs(x.astype(np.float32)), axis=1)
    assert np.all((codes[np.arange(len(x)), idx] & 0x7F) == 0x7B)


def test_e5m2_dequant_error_bound_per_element():
    # 2-bit mantissa: |q*s - x| <= max(2^-3 |x|, 2^-17 s) plus fp32 slack.
    rng = np.random.default_rng(39)
    x = (rng.standard_normal((64, 512)) * np.exp(rng.uniform(-4, 4, (64, 1)))).astype(np.float16)
    codes, s = quant_rows(x, "e5m2")
    deq = e5m2_decode(codes) * s.astype(np.float64)[:, None]
    xa = np.abs(x.astype(np.float64))
    bound = np.maximum(2.0 ** -3 * xa, 2.0 ** -17 * s.astype(np.float64)[:, None]) * (1 + 2.0 ** -18) + xa * 2.0 ** -20
    err = np.abs(deq - x.astype(np.float64))
    assert np.all(err <= bound)
    # and the E5M2 error is really coarser than E4M3's on the same rows
    c4, s4 = quant_rows(x)
    err4 = np.abs(e4m3_decode(c4) * s4.astype(np.float64)[:, None] - x.astype(np.float64))
    assert err.mean() > 1.5 * err4.mean()


def test_e5m2_brute_force_small_rows():
    finite = [c for c in range(256) if ((c >> 2) & 0x1F) != 31]
    table = {c: float(e5m2_decode(np.array([c], np.uint8))[0]) for c in finite}
    rng = np.random.default_rng(41)
    x = (rng.standard_normal((5, 40)) * 3).astype(np.float16)
    codes, s = quant_rows(x, "e5m2")
    for i in range(x.shape[0]):
        a = max(float(np.max(np.abs(x[i].astype(np.float32)))), float(EPS))
        r = np.float32(np.float32(57344.0) / np.float32(a))
        for k in range(x.shape[1]):
            t = float(np.float32(np.float32(x[i, k]) * r))
            t = min(max(t, -57344.0), 57344.0)
            best = min(finite, key=lambda c: (abs(table[c] - t), c & 1,
                                              (c >> 7) != (1 if np.signbit(t) else 0)))
            assert codes[i, k] == best or (t == 0.0 and (codes[i, k] & 0x7F) == 0), (i, k, t)


# ---------------------------------------------------------------------------
# Per-tensor weight scale (same page, §2.1: FFN linears quantized per tensor).

def test_per_tensor_one_scale_and_matches_rows_when_row_maxima_agree():
    rng = np.random.default_rng(45)
    w = (rng.standard_normal((24, 96)) * 0.02).astype(np.float16)
    w[:, 5] = np.float16(0.125)            # every row's amax is 0.125 (all |w| < 0.125 otherwise)
    w[:, 5][::2] = np.float16(-0.125)
    assert np.abs(w.astype(np.float32)).max() == np.float32(0.125)
    codes, s = quant_tensor(w)
    assert s.shape == (24,) and np.all(s == s[0])
    c_rows, s_rows = quant_rows(w)
    np.testing.assert_array_equal(codes, c_rows)
    np.testing.assert_array_equal(s, s_rows)


def test_per_tensor_uses_the_global_maximum():
    rng = np.random.default_rng(47)
    w = (rng.standard_normal((16, 64)) * np.linspace(0.01, 1.0, 16)[:, None]).astype(np.float16)
    codes, s = quant_tensor(w)
    a = np.float32(np.abs(w.astype(np.float32)).max())
    assert s[0] == np.float32(a / np.float32(448.0))
    big = int(np.argmax(np.abs(w.astype(np.float32)).max(axis=1)))
    # the row holding the global maximum is quantized exactly as by itself
    c_big, s_big = quant_rows(w[big:big + 1])
    np.testing.assert_array_equal(codes[big], c_big[0])
    # other rows use the larger shared scale: every code magnitude <= per-row code magnitude
    c_rows, _ = quant_rows(w)
    assert np.all(e4m3_decode(codes & 0x7F) <= e4m3_decode(c_rows & 0x7F))
    # dequantization error bound with the shared scale
    deq = e4m3_decode(codes) * np.float64(s[0])
    wa = np.abs(w.astype(np.float64))
    bound = np.maximum(2.0 ** -4 * wa, 2.0 ** -10 * np.float64(s[0])) * (1 + 2.0 ** -18) + wa * 2.0 ** -20
    assert np.all(np.abs(deq - w.astype(np.float64)) <= bound)


def test_per_tensor_zero_matrix_and_empty():
    codes, s = quant_tensor(np.zeros((3, 8), np.float16))
    assert np.all(codes == 0) and np.all(s == np.float32(EPS / np.float32(448.0)))
    c, s = quant_tensor(np.zeros((0, 8), np.float16))
    assert c.shape == (0, 8) and s.shape == (0,)
