"""The allocation-free entry point, fp8q_quantized_linear_noalloc.

Some callers cannot allocate device memory (a host framework that owns all of
it through its own pool, or a serving loop that must not allocate once it
runs).  This entry point keeps the codes and scales that pass between the
quantizer and the GEMM in a fixed scratch array inside the library instead
of a caller workspace.  The test calls it through the C ABI twice in a row,
on different shapes, and checks each result against the existing entry point
(fp8q_quantized_linear with a workspace) within the parity tolerance.  The
file is named to run last, so that a failure here stops a run only after
every other test has run.
"""
import pytest
import torch

from fp8_quantized_generative_b200 import _lib
from fp8_quantized_generative_b200 import workloads as wl

from parity import assert_close_f16, to_np

pytestmark = pytest.mark.gpu


def _existing(X, Wq, s_w, N):
    M, K = X.shape
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    Xq = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    s_x = torch.empty((M,), dtype=torch.float32, device="cuda")
    st = _lib.fp8q_quantized_linear(X.data_ptr(), Wq.data_ptr(), s_w.data_ptr(), M, N, K, Y.data_ptr(),
                                    Xq.data_ptr(), s_x.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == _lib.FP8Q_OK, _lib.last_error_message()
    return Y


def _noalloc(X, Wq, s_w, N):
    M, K = X.shape
    Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    st = _lib.fp8q_quantized_linear_noalloc(X.data_ptr(), Wq.data_ptr(), s_w.data_ptr(), M, N, K, Y.data_ptr(),
                                            torch.cuda.current_stream().cuda_stream)
    assert st == _lib.FP8Q_OK, _lib.last_error_message()
    return Y


def test_noalloc_matches_existing_entry_point_twice():
    import fp8_quantized_generative_b200 as fq
    # Largest first (it fills the scratch exactly: M*K = 8388608 codes), then
    # smaller shapes that reuse the same scratch, so codes or scales left over
    # from an earlier, larger call would show up; the last one (8 rows) runs
    # the split-K kernel, the others the CTA-pair kernel.
    cases = [(4096, 6144, 2048, 12), (300, 520, 1040, 11), (8, 4096, 4096, 13)]
    for M, N, K, seed in cases:
        X = wl.random_f16((M, K), seed=seed, std=2.0).cuda()
        Wq, s_w = fq.quantize_weight_per_channel(wl.random_f16((N, K), seed=seed + 1, std=0.02).cuda())
        y_ref = _existing(X, Wq, s_w, N)
        y_new = _noalloc(X, Wq, s_w, N)
        torch.cuda.synchronize()
        # the same kernels on the same inputs: bit for bit, and within the
        # path's tolerance of the oracle-checked entry point
        assert torch.equal(y_new.view(torch.int16), y_ref.view(torch.int16)), f"noalloc {M}x{N}x{K} not bitwise equal"
        assert_close_f16(to_np(y_new), to_np(y_ref), f"noalloc {M}x{N}x{K}")
    assert fq.device_error() == 0


def test_noalloc_rejects_sizes_beyond_the_scratch():
    a = 0x1000
    st = _lib.fp8q_quantized_linear_noalloc(a, a, a, 4097, 16, 2048, a, 0)   # M*K > 8 Mi
    assert st == _lib.FP8Q_ERR_INVALID_ARG
    assert "8388608" in _lib.last_error_message()
    st = _lib.fp8q_quantized_linear_noalloc(a, a, a, 16385, 16, 16, a, 0)    # M > 16384 scales
    assert st == _lib.FP8Q_ERR_INVALID_ARG
    assert "16384" in _lib.last_error_message()
