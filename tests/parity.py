"""Shared helpers for the GPU-vs-oracle parity tests.

Tolerance for FP16 outputs (FP32 accumulation order is hardware-defined, so
outputs are not bit-pinned; codes and scales are):
    per element:  |Y_gpu - Y_ref| <= 2^-9 * |Y_ref| + 1e-3 * rms(Y_ref)
    whole tensor: ||Y_gpu - Y_ref||_F / ||Y_ref||_F <= 1e-3
"""
import numpy as np
import torch

REL_ELEM = 2.0 ** -9
ABS_RMS = 1e-3
REL_FRO = 1e-3


def assert_close_f16(y_gpu, y_ref, what=""):
    g = np.asarray(y_gpu, dtype=np.float64)
    r = np.asarray(y_ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    if r.size == 0:
        return
    rms = float(np.sqrt(np.mean(r * r)))
    err = np.abs(g - r)
    bound = REL_ELEM * np.abs(r) + ABS_RMS * rms
    bad = err > bound
    if np.any(bad):
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance; first at {tuple(i)}: "
                             f"gpu={g[tuple(i)]!r} ref={r[tuple(i)]!r} bound={bound[tuple(i)]!r}")
    fro = np.linalg.norm(r)
    if fro > 0:
        rel = np.linalg.norm(g - r) / fro
        assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"


def sample_rows(M, n, seed=0):
    """Up to n row indices spread over [0, M): always the first and last rows."""
    if M <= n:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, M - 1), size=n - 2, replace=False)
    return np.sort(np.concatenate([[0, M - 1], mid]))


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def assert_no_device_error():
    import fp8_quantized_generative_b200 as fq
    flags = fq.device_error()
    assert flags == 0, f"device error word 0x{flags:x}"
