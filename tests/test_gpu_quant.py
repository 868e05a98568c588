"""GPU parity of the per-row E4M3 quantizer and the device cast: bit-exact.

Codes and scales from libfp8q are compared byte for byte with the CPU oracle
(oracle.quant_rows / oracle.e4m3_encode) on the same seeded inputs: every row
of every matrix, the full-size ones included, with guard-banded outputs.  The
device cast is swept over all 2^32 fp32 bit patterns (test_zy_cast_sweep.py).
"""
import numpy as np
import pytest
import torch

from oracle import e4m3_encode, quant_rows
from fp8_quantized_generative_b200 import workloads as wl

from parity import Guards, assert_no_device_error, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import fp8_quantized_generative_b200 as m
    assert torch.cuda.is_available()
    return m


def _check_rows(fq, X, what=""):
    Xd = X.cuda()
    # sentinel-filled, guard-banded outputs: unwritten codes or scales fail
    # the comparison, writes past either end fail the guard check
    g = Guards()
    Xq = g(X.shape, torch.uint8, 0x7F, "Xq")
    s = g((X.shape[0],), torch.float32, float("nan"), "s")
    fq.quantize_rows_dynamic(Xd, out=(Xq, s))
    g.check(what)
    ref_q, ref_s = quant_rows(X.numpy())
    got_q = to_np(Xq)
    got_s = to_np(s)
    if not np.array_equal(got_q, ref_q):
        bad = np.argwhere(got_q != ref_q)[0]
        raise AssertionError(f"{what}: code mismatch at {tuple(bad)}: gpu 0x{got_q[tuple(bad)]:02x} "
                             f"oracle 0x{ref_q[tuple(bad)]:02x}")
    np.testing.assert_array_equal(got_s.view(np.uint32), ref_s.view(np.uint32), err_msg=what)
    assert_no_device_error()


def test_tiny_activations_and_weights(fq):
    lin = wl.tiny()
    _check_rows(fq, lin.X, what="tiny X")
    _check_rows(fq, lin.W, what="tiny W")


@pytest.mark.parametrize("M,K", [(1, 16), (3, 272), (37, 1024), (129, 2064), (5, 4096), (9, 8192), (2, 24576),
                                 (260, 256)])
def test_ragged_shapes(fq, M, K):
    X = wl.random_f16((M, K), seed=M * 7 + K, std=3.0)
    _check_rows(fq, X, what=f"{M}x{K}")


def test_edge_rows(fq):
    K = 512
    X = wl.random_f16((6, K), seed=5).float()
    X[0] = 0.0                            # all-zero row -> eps scale
    X[1, 17] = 65504.0                    # fp16 max
    X[2] = X[2] * 1e-4                    # small values, subnormal codes
    X[3, :] = 448.0                       # exact unit scale
    X[4, ::2] = -0.0                      # negative zeros
    X[5] = 2.0 ** -24                     # fp16 subnormal magnitudes
    _check_rows(fq, X.to(torch.float16), what="edge rows")


def test_full_size_activations(fq):
    # every row of every full-size activation and weight matrix, bit for bit
    lin = wl.qkv()
    _check_rows(fq, lin.X, what="qkv X")
    _check_rows(fq, lin.W, what="qkv W")
    up, down = wl.ffn()
    _check_rows(fq, up.X, what="ffn_up X")
    _check_rows(fq, down.X, what="ffn_down X")
    _check_rows(fq, down.W, what="ffn_down W")
    for m in (1, 8, 128, 16384):
        _check_rows(fq, wl.sweep_x(m), what=f"sweep X m={m}")


def test_moe_weights_per_channel(fq):
    m = wl.moe()
    Wd = m.W_up.cuda()
    Wq, s = fq.quantize_weight_per_channel(Wd)
    torch.cuda.synchronize()
    assert Wq.shape == m.W_up.shape and s.shape == m.W_up.shape[:2]
    E, N, K = m.W_up.shape
    ref_q, ref_s = quant_rows(m.W_up.reshape(E * N, K).numpy())
    np.testing.assert_array_equal(to_np(Wq).reshape(E * N, K), ref_q)
    np.testing.assert_array_equal(to_np(s).reshape(E * N).view(np.uint32), ref_s.view(np.uint32))
    assert_no_device_error()


def _stratified_patterns():
    tails = np.array([0, 1, 2, 0x3FFF, 0x4000, 0x4001, 0x7FFF, 0x2000, 0x5555, 0x7FFE, 0x0800, 0x6000],
                     dtype=np.uint32)
    exps = np.arange(256, dtype=np.uint32) << 23
    heads = np.arange(256, dtype=np.uint32) << 15
    bits = (exps[:, None, None] | heads[None, :, None] | tails[None, None, :]).reshape(-1)
    return np.concatenate([bits, bits | np.uint32(0x80000000)])


def test_device_cast_against_oracle(fq):
    rng = np.random.default_rng(123)
    bits = np.concatenate([
        _stratified_patterns(),
        rng.integers(0, 2 ** 32, size=8_000_000, dtype=np.uint64).astype(np.uint32),
        np.arange(2 ** 16, dtype=np.uint16).view(np.float16).astype(np.float32).view(np.uint32),
    ])
    v = bits.view(np.float32)
    v = v[~np.isnan(v)]                      # NaN inputs are outside the contract
    got = to_np(fq.e4m3_encode_f32(torch.from_numpy(v).cuda()))
    ref = e4m3_encode(v)
    if not np.array_equal(got, ref):
        i = int(np.argwhere(got != ref)[0][0])
        raise AssertionError(f"cast mismatch for {v[i]!r} (bits 0x{v.view(np.uint32)[i]:08x}): "
                             f"gpu 0x{got[i]:02x} oracle 0x{ref[i]:02x}")
    # odd length exercises the tail element
    got = to_np(fq.e4m3_encode_f32(torch.tensor([1.0, -3.5, 500.0], device="cuda")))
    np.testing.assert_array_equal(got, e4m3_encode(np.array([1.0, -3.5, 500.0], np.float32)))


def test_quantize_is_deterministic(fq):
    X = wl.random_f16((333, 1024), seed=9).cuda()
    a = fq.quantize_rows_dynamic(X)
    b = fq.quantize_rows_dynamic(X)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
