"""Pins for the oracle's per-row quantization (per-token / per-channel scales).

Rule under test ('Quantized Inference for OneRec-V2', 关键证据 steps 1-2;
'FP8量化在生成式推荐系统OneRec-V2中的优化实践' §2.2 scale = max_code / max(|x|, eps)):
    a' = max(max|x|, 1e-12); r = fl32(448/a'); s = fl32(a'/448); q = E4M3(fl32(x*r)).
"""
import json
import os

import numpy as np
import pytest

from oracle import EPS, e4m3_decode, quant_rows


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
