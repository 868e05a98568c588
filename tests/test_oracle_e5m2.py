"""Pins for the oracle's E5M2 codec (the activation format variant).

'FP8量化在生成式推荐系统OneRec-V2中的优化实践' §2.2 names E5M2 (5 exponent bits,
2 mantissa bits) for activations.  The codec is checked against things other
than itself:
  * the closed form of the format (bias 15, largest finite 1.75 * 2^15 = 57344,
    smallest normal 2^-14, smallest subnormal 2^-16, infinities and NaNs);
  * PyTorch's float8_e5m2 conversion, an independent library routine
    (round-to-nearest-even; it overflows to infinity from 61440 up, so
    saturation is pinned separately);
  * the round-trip error bound of a 2-bit mantissa (2^-3 relative on normals,
    2^-17 absolute on subnormals) and ties-to-even at every midpoint.
"""
import numpy as np
import torch

from oracle import e5m2_decode, e5m2_encode


def torch_e5m2_codes(v32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(v32, dtype=np.float32))
    return t.to(torch.float8_e5m2).view(torch.uint8).numpy()


ALL_CODES = np.arange(256, dtype=np.uint8)
_EXP = (ALL_CODES >> 2) & 0x1F
FINITE = ALL_CODES[_EXP != 31]


def test_decode_closed_form_points():
    d = e5m2_decode(np.array([0x7B, 0xFB, 0x04, 0x01, 0x03, 0x00, 0x80, 0x3C, 0x3D], dtype=np.uint8))
    assert d[0] == 57344.0 and d[1] == -57344.0      # 1.75 * 2^15
    assert d[2] == 2.0 ** -14                        # smallest normal
    assert d[3] == 2.0 ** -16                        # smallest subnormal
    assert d[4] == 3 * 2.0 ** -16                    # largest subnormal
    assert d[5] == 0.0 and d[6] == 0.0 and np.signbit(d[6])
    assert d[7] == 1.0 and d[8] == 1.25              # exponent field 15 = bias
    specials = e5m2_decode(np.array([0x7C, 0xFC, 0x7D, 0x7E, 0x7F, 0xFF], dtype=np.uint8))
    assert specials[0] == np.inf and specials[1] == -np.inf
    assert np.isnan(specials[2:]).all()


def test_decode_matches_library_table():
    ref = torch.from_numpy(ALL_CODES.copy()).view(torch.float8_e5m2).to(torch.float64).numpy()
    ours = e5m2_decode(ALL_CODES)
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[fin], ref[fin])
    np.testing.assert_array_equal(np.signbit(ours[fin]), np.signbit(ref[fin]))


def test_decode_is_monotone_over_positive_codes():
    pos = e5m2_decode(np.arange(0, 0x7C, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)


def test_encode_decode_identity_on_finite_codes():
    vals = e5m2_decode(FINITE).astype(np.float32)
    np.testing.assert_array_equal(e5m2_encode(vals), FINITE)


def test_negative_zero_and_nan():
    assert e5m2_encode(np.float32(-0.0)) == 0x80
    assert e5m2_encode(np.float32(0.0)) == 0x00
    assert e5m2_encode(np.float32(np.nan)) == 0x7F


def test_saturation_never_reaches_infinity():
    big = np.array([57344.0, 57344.5, 61439.0, 61440.0, 65504.0, 1e9, 3.4e38, np.inf], dtype=np.float32)
    np.testing.assert_array_equal(e5m2_encode(big), np.full(big.shape, 0x7B, np.uint8))
    np.testing.assert_array_equal(e5m2_encode(-big), np.full(big.shape, 0xFB, np.uint8))


def stratified_f32_patterns() -> np.ndarray:
    """Every float32 exponent x every top-8 mantissa prefix x low-bit tails that
    put the E5M2 round bit (mantissa bit 20) below, at and above half-way."""
    tails = np.array([0, 1, 0x1FFFF, 0x20000, 0x20001, 0x3FFFF, 0x10000, 0x0FFFF, 0x2AAAA], dtype=np.uint32)
    exps = np.arange(256, dtype=np.uint32) << 23
    heads = np.arange(64, dtype=np.uint32) << 17
    bits = (exps[:, None, None] | heads[None, :, None] | tails[None, None, :]).reshape(-1)
    bits = np.concatenate([bits, bits | np.uint32(0x80000000)])
    return bits.view(np.float32)


def _check_against_library(v: np.ndarray):
    v = v[~np.isnan(v)]
    small = np.abs(v.astype(np.float64)) < 61440.0
    np.testing.assert_array_equal(e5m2_encode(v[small]), torch_e5m2_codes(v[small]))
    big = v[~small]
    np.testing.assert_array_equal(e5m2_encode(big), np.where(np.signbit(big), 0xFB, 0x7B).astype(np.uint8))


def test_encode_stratified_against_library():
    _check_against_library(stratified_f32_patterns())


def test_encode_random_bits_against_library():
    rng = np.random.default_rng(17)
    bits = rng.integers(0, 2 ** 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    _check_against_library(bits.view(np.float32))


def test_encode_all_fp16_values_against_library():
    v = np.arange(2 ** 16, dtype=np.uint16).view(np.float16).astype(np.float32)
    _check_against_library(v)


def test_round_trip_bound():
    rng = np.random.default_rng(21)
    t = np.concatenate([
        np.exp(rng.uniform(np.log(2.0 ** -14), np.log(57344.0), 1_000_000)),
        rng.uniform(0, 2.0 ** -14, 200_000),
    ]).astype(np.float32)
    t = np.concatenate([t, -t])
    back = e5m2_decode(e5m2_encode(t))
    err = np.abs(back - t.astype(np.float64))
    a = np.abs(t.astype(np.float64))
    normal = a >= 2.0 ** -14
    assert np.all(err[normal] <= 2.0 ** -3 * a[normal])
    assert np.all(err[~normal] <= 2.0 ** -17)


def test_round_to_nearest_even_midpoints():
    pos = e5m2_decode(np.arange(0, 0x7C, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    assert np.all(mids.astype(np.float64) == (pos[:-1] + pos[1:]) / 2)   # exact in fp32
    codes = e5m2_encode(mids).astype(np.int64)
    lower = np.arange(0, 0x7B)
    np.testing.assert_array_equal(codes, np.where(lower % 2 == 0, lower, lower + 1))
