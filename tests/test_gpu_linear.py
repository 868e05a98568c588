"""GPU parity of the FP8 W8A8 linear (quantize + tcgen05 GEMM + fused dequant).

Each case draws seeded fp16 X and W, runs the library path (per-token
quantization, per-channel weight quantization, fp8q_linear) and compares the
fp16 output with the CPU oracle (quant_rows + linear_ref in float64) computed
from the same fp16 inputs, element by element over the WHOLE output, at every
size including the full workloads (the float64 oracle is a BLAS matmul, so
the largest case costs seconds on the host).  The codes and scales of the
intermediate quantization are compared bit for bit as well.

Every device output (Wq, s_w, Xq, s_x, Y) lives inside a guard-banded buffer
(4 KiB of a seeded byte pattern on each side, checked after the call): a
kernel that writes past either end of an output fails the test.  Outputs
start NaN (or 0xFF codes, which finite inputs never produce), so an element
that no kernel writes fails the comparison.
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


def run_gpu(fq, X, W, guards=None):
    g = guards if guards is not None else Guards()
    M, K = X.shape
    N = W.shape[0]
    Xd, Wd = X.cuda(), W.cuda()
    Wq = g((N, K), torch.uint8, 0xFF, "Wq")
    s_w = g((N,), torch.float32, float("nan"), "s_w")
    fq.quantize_weight_per_channel(Wd, out=(Wq, s_w))
    Xq = g((M, K), torch.uint8, 0xFF, "Xq")
    s_x = g((M,), torch.float32, float("nan"), "s_x")
    fq.quantize_rows_dynamic(Xd, out=(Xq, s_x))
    # NaN-filled output: any element the kernel fails to write fails the check
    Y = g((M, N), torch.float16, float("nan"), "Y")
    fq.linear(Xq, s_x, Wq, s_w, out=Y)
    torch.cuda.synchronize()
    g.check(f"{M}x{N}x{K}")
    return Y, (Xq, s_x, Wq, s_w)


def oracle_all(X, W):
    Wq, s_w = quant_rows(W.numpy())
    Xq, s_x = quant_rows(X.numpy())
    return linear_ref(Xq, s_x, Wq, s_w), (Xq, s_x, Wq, s_w)


def check(fq, X, W, what=""):
    Y, got = run_gpu(fq, X, W)
    ref, exp = oracle_all(X, W)
    for name, a, b in zip(("Xq", "s_x", "Wq", "s_w"), got, exp):
        a = to_np(a)
        if a.dtype == np.float32:
            a, b = a.view(np.uint32), b.view(np.uint32)
        if not np.array_equal(a, b):
            i = tuple(np.argwhere(a != b)[0])
            raise AssertionError(f"{what}: {name} differs from the oracle at {i}: {a[i]!r} vs {b[i]!r}")
    assert_close_f16(to_np(Y), ref, what)
    assert_no_device_error()
    return Y


def test_tiny(fq):
    lin = wl.tiny()
    check(fq, lin.X, lin.W, what="tiny")


@pytest.mark.parametrize("M,N,K", [
    (1, 256, 128), (128, 256, 128), (300, 520, 272), (257, 264, 1040), (77, 1000, 16), (1000, 8, 64),
    (640, 768, 4096),
])
def test_ragged_and_multi_tile(fq, M, N, K):
    X = wl.random_f16((M, K), seed=M + N + K)
    W = wl.random_f16((N, K), seed=M * N + K, std=0.02)
    check(fq, X, W, what=f"{M}x{N}x{K}")


def test_edge_values(fq):
    K, N = 256, 256
    X = wl.random_f16((8, K), seed=3).float()
    X[0] = 0.0                  # zero row -> zero output row
    X[1, 5] = 65504.0           # huge outlier
    X[2] = 448.0
    W = wl.random_f16((N, K), seed=4, std=0.02).float()
    W[7] = 0.0                  # zero channel
    Y = check(fq, X.half(), W.half(), what="edge")
    y = to_np(Y).astype(np.float64)
    assert np.all(y[0] == 0) and np.all(y[:, 7] == 0)


def test_qkv_full(fq):
    lin = wl.qkv()
    check(fq, lin.X, lin.W, what="qkv 4096x6144x2048")


def test_ffn_full(fq):
    up, down = wl.ffn()
    check(fq, up.X, up.W, what="ffn up 8192x8192x2048")
    check(fq, down.X, down.W, what="ffn down 8192x2048x8192")


@pytest.mark.parametrize("m", wl.SWEEP_M)
def test_sweep(fq, m):
    check(fq, wl.sweep_x(m), wl.sweep_w(), what=f"sweep m={m}")


def test_deterministic(fq):
    lin = wl.qkv(m=512)
    a, _ = run_gpu(fq, lin.X, lin.W)
    b, _ = run_gpu(fq, lin.X, lin.W)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_zero_rows_noop(fq):
    Xq = torch.empty((0, 128), dtype=torch.uint8, device="cuda")
    s = torch.empty((0,), dtype=torch.float32, device="cuda")
    Wq = torch.zeros((64, 128), dtype=torch.uint8, device="cuda")
    sw = torch.ones((64,), dtype=torch.float32, device="cuda")
    Y = fq.linear(Xq, s, Wq, sw)
    assert Y.shape == (0, 64)


VARIANTS = [(1, 0), (2, 128), (2, 192), (2, 256), (2, 512)]


@pytest.mark.parametrize("family,bn", VARIANTS)
@pytest.mark.parametrize("M,N,K", [(300, 520, 272), (257, 1000, 1040), (1024, 6144, 2048), (512, 768, 128)])
def test_kernel_variants(fq, family, bn, M, N, K):
    X = wl.random_f16((M, K), seed=M + 3 * N + K)
    W = wl.random_f16((N, K), seed=N + K, std=0.02)
    fq.set_gemm_tuning(family, bn)
    try:
        check(fq, X, W, what=f"family={family} bn={bn} {M}x{N}x{K}")
    finally:
        fq.set_gemm_tuning(0, 0, 0)


@pytest.mark.parametrize("ksplit", [1, 2, 4, 8])
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (5, 264, 272), (16, 1000, 2048), (33, 520, 1040),
                                   (64, 256, 128), (100, 6144, 2048), (128, 4096, 4096)])
def test_splitk_variants(fq, ksplit, M, N, K):
    X = wl.random_f16((M, K), seed=7 * M + N + K)
    W = wl.random_f16((N, K), seed=N + 2 * K, std=0.02)
    fq.set_gemm_tuning(3, 0, ksplit)
    try:
        check(fq, X, W, what=f"splitk S={ksplit} {M}x{N}x{K}")
    finally:
        fq.set_gemm_tuning(0, 0, 0)


def test_split_k_stage_forms_in_a_subprocess():
    # The split-K kernel (M <= 128) runs four-box (512-byte) stages up to 32
    # rows and two-box (256-byte) stages above; the one-box form stays
    # selectable.  Each form is forced for every row count here
    # (FP8Q_SPLITK_STAGE_K is read once per process; 512 falls back to two
    # boxes above 32 rows) and checked against the oracle, including ragged
    # K and a forced split of 8.
    import os
    import subprocess
    import sys
    code = r'''
import sys, torch
sys.path.insert(0, "tests")
from test_gpu_linear import check
import fp8_quantized_generative_b200 as fq
from fp8_quantized_generative_b200 import workloads as wl
for M, N, K in [(1, 4096, 4096), (16, 1000, 2048), (33, 520, 1040), (100, 6144, 2048), (128, 264, 272)]:
    for ks in (0, 8):
        fq.set_gemm_tuning(3, 0, ks)
        check(fq, wl.random_f16((M, K), seed=M + K), wl.random_f16((N, K), seed=N, std=0.02), what=f"{M}x{N}x{K} S={ks}")
print("ok")
'''
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for sk in ("128", "256", "512"):
        env = dict(os.environ, FP8Q_SPLITK_STAGE_K=sk)
        r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True, text=True, timeout=600)
        assert r.returncode == 0 and r.stdout.strip().endswith("ok"), sk + r.stdout[-2000:] + r.stderr[-2000:]


def test_one_box_stages_path_in_a_subprocess():
    # The dense CTA-pair kernel runs 256-byte K stages by default; the
    # one-box (128-byte) stage form stays selectable (FP8Q_STAGE_K=128, read
    # once per process), so it is checked against the oracle in a process of
    # its own, on ragged and multi-round shapes.
    import os
    import subprocess
    import sys
    code = r'''
import sys, torch
sys.path.insert(0, "tests")
from test_gpu_linear import check
import fp8_quantized_generative_b200 as fq
from fp8_quantized_generative_b200 import workloads as wl
for M, N, K in [(300, 520, 272), (1024, 6144, 2048), (257, 1000, 1040)]:
    check(fq, wl.random_f16((M, K), seed=M + K), wl.random_f16((N, K), seed=N, std=0.02), what=f"{M}x{N}x{K}")
print("ok")
'''
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, FP8Q_STAGE_K="128")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-2000:]
