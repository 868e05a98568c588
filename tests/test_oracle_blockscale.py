"""Pins for the oracle's block-wise weight quantization and block-scaled linear
('FP8量化在生成式推荐系统OneRec-V2中的优化实践' §2.1: the MoE expert grouped GEMM is
quantized block-wise 128x128; §2.2: block-aligned MoE quantization;
activations stay per token).

  * a hand-worked case with 2x2 blocks (tests/golden/quant_blocks_hand.json);
  * every block equals the per-tensor quantization of that block alone, and
    uniform block maxima reduce it to the per-tensor quantization of the whole
    matrix (quant_tensor is pinned on its own);
  * exactness: blocks whose entries are E4M3 values x 2^j_b with block
    maximum 448 * 2^j_b (a different j per block) quantize exactly, so the
    linear equals fp16(X @ W^T) bit for bit;
  * equal scales along K reduce the block-scaled linear to the per-channel one;
  * a brute-force error bound against the unquantized float64 product, tight
    enough to catch a transposed block-scale index.
"""
import json
import os

import numpy as np
import pytest

from oracle import (e4m3_decode, linear_blockscaled_ref, linear_f64_unquantized, linear_ref, moe_blockscaled_ref,
                    quant_blocks, quant_rows, quant_tensor)

FINITE_POS = e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))


def test_hand_worked_blocks(golden_dir):
    with open(os.path.join(golden_dir, "quant_blocks_hand.json")) as f:
        case = json.load(f)
    b = case["block"]
    W = np.array([[np.float16(v) for v in r] for r in case["W"]], dtype=np.float16)
    codes, s = quant_blocks(W, block=b)
    np.testing.assert_array_equal(codes, np.array([[int(c, 16) for c in r] for r in case["codes"]], np.uint8))
    np.testing.assert_array_equal(s.view(np.uint32),
                                  np.array([[int(c, 16) for c in r] for r in case["scale_f32_bits"]], np.uint32))
    X = np.array([[np.float16(v) for v in r] for r in case["X"]], dtype=np.float16)
    xq, sx = quant_rows(X)
    Y = linear_blockscaled_ref(xq, sx, codes, s, block=b)
    np.testing.assert_array_equal(Y[0].astype(np.float64), np.array([float(v) for v in case["Y"]]))


@pytest.mark.parametrize("R,K,b", [(300, 272, 128), (17, 33, 8), (128, 128, 128)])
def test_each_block_is_its_own_per_tensor_quantization(R, K, b):
    rng = np.random.default_rng(R + K)
    W = (rng.standard_normal((R, K)) * np.exp(rng.uniform(-3, 3, (R, 1)))).astype(np.float16)
    codes, s = quant_blocks(W, block=b)
    assert s.shape == (-(-R // b), -(-K // b))
    for i in range(s.shape[0]):
        for j in range(s.shape[1]):
            blk = W[i * b:(i + 1) * b, j * b:(j + 1) * b]
            c_t, s_t = quant_tensor(blk)
            np.testing.assert_array_equal(codes[i * b:(i + 1) * b, j * b:(j + 1) * b], c_t)
            assert s[i, j] == s_t[0]


def test_uniform_block_maxima_reduce_to_per_tensor():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((256, 384)) * 0.02).astype(np.float16)
    W[::128, ::128] = np.float16(0.5)            # every 128x128 block holds the global maximum 0.5
    assert np.abs(W.astype(np.float32)).max() == np.float32(0.5)
    c_b, s_b = quant_blocks(W)
    c_t, s_t = quant_tensor(W)
    np.testing.assert_array_equal(c_b, c_t)
    assert np.all(s_b == s_t[0])


def exact_block_matrix(rng, rows, cols, b, js):
    """Blocks of E4M3 values x 2^j_b with one ±448*2^j_b per block; js [ceil(rows/b), ceil(cols/b)]."""
    v = rng.choice(FINITE_POS, size=(rows, cols)) * rng.choice([-1.0, 1.0], size=(rows, cols))
    m = np.zeros((rows, cols))
    for i in range(js.shape[0]):
        for j in range(js.shape[1]):
            blk = v[i * b:(i + 1) * b, j * b:(j + 1) * b].copy()
            blk.flat[rng.integers(0, blk.size)] = 448.0 * rng.choice([-1.0, 1.0])
            m[i * b:(i + 1) * b, j * b:(j + 1) * b] = blk * 2.0 ** js[i, j]
    out = m.astype(np.float16)
    assert np.all(out.astype(np.float64) == m)
    return out


@pytest.mark.parametrize("M,N,K,b", [(7, 20, 40, 8), (5, 256, 384, 128)])
def test_exactness_with_per_block_powers_of_two(M, N, K, b):
    rng = np.random.default_rng(M * 31 + N)
    js = rng.integers(-10, -5, size=(-(-N // b), -(-K // b)))
    W = exact_block_matrix(rng, N, K, b, js)
    # activations: E4M3 values x 2^-3 with every row's maximum ±448 * 2^-3 (exact per-token scales)
    xv = rng.choice(FINITE_POS, size=(M, K)) * rng.choice([-1.0, 1.0], size=(M, K))
    xv[np.arange(M), rng.integers(0, K, M)] = 448.0 * rng.choice([-1.0, 1.0], size=M)
    X = (xv * 2.0 ** -3).astype(np.float16)
    assert np.all(X.astype(np.float64) == xv * 2.0 ** -3)
    Xq, sx = quant_rows(X)
    Wq, swb = quant_blocks(W, block=b)
    np.testing.assert_array_equal(swb, (2.0 ** js).astype(np.float32))
    np.testing.assert_array_equal(e4m3_decode(Wq) * np.repeat(np.repeat(2.0 ** js, b, 0), b, 1)[:N, :K],
                                  W.astype(np.float64))
    Y = linear_blockscaled_ref(Xq, sx, Wq, swb, block=b)
    expect = (X.astype(np.float64) @ W.astype(np.float64).T).astype(np.float16)
    np.testing.assert_array_equal(Y.view(np.uint16), expect.view(np.uint16))


def test_equal_scales_along_k_reduce_to_per_channel():
    rng = np.random.default_rng(9)
    b = 16
    N, K, M = 48, 64, 6
    js = np.repeat(rng.integers(-9, -6, size=(N // b, 1)), K // b, axis=1)      # one scale per row block
    W = exact_block_matrix(rng, N, K, b, js)
    X = rng.standard_normal((M, K)).astype(np.float16)
    Xq, sx = quant_rows(X)
    Wq, swb = quant_blocks(W, block=b)
    s_rows = np.repeat(swb[:, 0], b)[:N]
    np.testing.assert_array_equal(linear_blockscaled_ref(Xq, sx, Wq, swb, block=b).view(np.uint16),
                                  linear_ref(Xq, sx, Wq, s_rows).view(np.uint16))


def block_error_bound(X, W, sx, swb, b, Y):
    xa = np.abs(X.astype(np.float64))
    wa = np.abs(W.astype(np.float64))
    N, K = W.shape
    sw_elem = np.repeat(np.repeat(swb.astype(np.float64), b, 0), b, 1)[:N, :K]
    dx = np.maximum(2.0 ** -4 * xa, 2.0 ** -10 * sx.astype(np.float64)[:, None]) * (1 + 2.0 ** -18) + xa * 2.0 ** -20
    dw = np.maximum(2.0 ** -4 * wa, 2.0 ** -10 * sw_elem) * (1 + 2.0 ** -18) + wa * 2.0 ** -20
    prod = (xa + dx) @ (wa + dw).T - xa @ wa.T
    return prod * (1 + 2.0 ** -40) + 2.0 ** -10 * np.abs(Y.astype(np.float64)) + 2.0 ** -24


@pytest.mark.parametrize("seed", range(4))
def test_brute_force_error_bound(seed):
    rng = np.random.default_rng(500 + seed)
    b = 8
    M, N, K = rng.integers(1, 12), rng.integers(1, 30), rng.integers(1, 40)
    X = (rng.standard_normal((M, K)) * np.exp(rng.uniform(-2, 2, (M, 1)))).astype(np.float16)
    W = (rng.standard_normal((N, K)) * 0.02 * np.exp(rng.uniform(-2, 2, (N, K)))).astype(np.float16)
    Xq, sx = quant_rows(X)
    Wq, swb = quant_blocks(W, block=b)
    Y = linear_blockscaled_ref(Xq, sx, Wq, swb, block=b)
    err = np.abs(Y.astype(np.float64) - linear_f64_unquantized(X, W))
    assert np.all(err <= block_error_bound(X, W, sx, swb, b, Y))


def test_bound_catches_a_transposed_block_scale():
    rng = np.random.default_rng(77)
    b = 8
    X = rng.standard_normal((4, 32)).astype(np.float16)
    W = (rng.standard_normal((32, 32)) * np.exp(rng.uniform(-3, 3, (32, 32)))).astype(np.float16)
    Xq, sx = quant_rows(X)
    Wq, swb = quant_blocks(W, block=b)
    wrong = linear_blockscaled_ref(Xq, sx, Wq, swb.T.copy(), block=b)
    assert np.any(np.abs(wrong.astype(np.float64) - linear_f64_unquantized(X, W))
                  > block_error_bound(X, W, sx, swb, b, wrong))


def test_moe_single_expert_equals_dense_and_groups_are_independent():
    rng = np.random.default_rng(12)
    E, N, K, b = 3, 24, 40, 8
    counts = [4, 0, 6]
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    X = rng.standard_normal((10, K)).astype(np.float16)
    W = (rng.standard_normal((E, N, K)) * 0.05).astype(np.float16)
    Xq, sx = quant_rows(X)
    q = [quant_blocks(W[e], block=b) for e in range(E)]
    Wq = np.stack([c for c, _ in q])
    swb = np.stack([s for _, s in q])
    Y = moe_blockscaled_ref(Xq, sx, off, Wq, swb, block=b)
    for e in range(E):
        lo, hi = off[e], off[e + 1]
        np.testing.assert_array_equal(Y[lo:hi], linear_blockscaled_ref(Xq[lo:hi], sx[lo:hi], Wq[e], swb[e], block=b))
