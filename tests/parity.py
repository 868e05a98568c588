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


class Guarded:
    """A device tensor placed in the middle of a larger byte buffer whose
    `pad` bytes on either side hold a seeded byte pattern.

    Stands in for a memory checker: a kernel that writes past either end of
    the tensor changes the pattern, and check() reports it.  The interior
    starts `pad` bytes (a multiple of 256) into the allocation, so it keeps
    the 16-byte alignment the library requires.
    """

    def __init__(self, shape, dtype, fill=None, pad=4096, seed=0, device="cuda"):
        assert pad % 256 == 0
        self.pad = pad
        esize = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(shape)) if len(shape) else 1
        self.nbytes = n * esize
        g = torch.Generator().manual_seed(1000 + seed)
        total = 2 * pad + self.nbytes
        self.pattern = torch.randint(0, 256, (total,), generator=g, dtype=torch.uint8).to(device)
        self.buf = self.pattern.clone()
        inner = self.buf[pad:pad + self.nbytes]
        self.t = inner.view(dtype).view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self, what=""):
        lo = self.buf[:self.pad]
        hi = self.buf[self.pad + self.nbytes:]
        for name, got, exp in (("before", lo, self.pattern[:self.pad]),
                               ("after", hi, self.pattern[self.pad + self.nbytes:])):
            bad = (got != exp).nonzero()
            if bad.numel():
                first = int(bad[0, 0]) if name == "after" else int(bad[-1, 0]) - self.pad
                raise AssertionError(f"{what}: {bad.numel()} guard bytes {name} the tensor were overwritten "
                                     f"(nearest at byte offset {first} from its {'end' if name == 'after' else 'start'})")


class Guards:
    """Factory of Guarded tensors that checks all of them at once."""

    def __init__(self):
        self.items = []

    def __call__(self, shape, dtype, fill=None, name=""):
        g = Guarded(tuple(shape), dtype, fill, seed=len(self.items))
        self.items.append((name or f"tensor {len(self.items)}", g))
        return g.t

    def check(self, what=""):
        torch.cuda.synchronize()
        for name, g in self.items:
            g.check(f"{what} {name}".strip())


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def assert_no_device_error():
    import fp8_quantized_generative_b200 as fq
    flags = fq.device_error()
    assert flags == 0, f"device error word 0x{flags:x}"
