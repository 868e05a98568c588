"""The device E4M3 cast against the oracle's encoder on ALL 2^32 fp32 bit
patterns.

The quantizers' cast (round to nearest even, saturating to ±448; E4M3 as the
format of 'FP8量化在生成式推荐系统OneRec-V2中的优化实践' §2.2 with the range of
§1.2) is exposed alone as fp8q_e4m3_encode_f32.  Every fp32 pattern goes
through it on the GPU, 2^28 at a time, and through oracle.e4m3_encode on the
host cores (a spawned process pool: the oracle is plain NumPy, one process
per core), 2^24 at a time.  Each 2^24-pattern slice is compared by a BLAKE2b
digest of its codes; a differing slice is recomputed to name the first
differing pattern.  NaN inputs are outside the contract: their codes are
masked out of the digests, and the device must still return a NaN code for
them.  The oracle's encoder is itself pinned to the library float8_e4m3fn
cast over the same 2^32 patterns (tests/test_oracle_e4m3.py, opt-in).
"""
import hashlib
import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

import cast_sweep_worker as worker

pytestmark = pytest.mark.gpu

SLICE = 1 << 24          # patterns per digest
GPU_CHUNK = 1 << 28      # patterns per device call


def test_device_cast_all_fp32_patterns():
    import fp8_quantized_generative_b200 as fq
    assert torch.cuda.is_available()
    n_slices = (1 << 32) // SLICE
    procs = max(1, min(os.cpu_count() or 1, 32))
    ctx = mp.get_context("spawn")
    with ctx.Pool(procs) as pool:
        pending = pool.starmap_async(worker.digest, [(i * SLICE, (i + 1) * SLICE) for i in range(n_slices)],
                                     chunksize=1)
        gpu_digests = []
        idx = torch.arange(GPU_CHUNK, dtype=torch.int64, device="cuda")
        for lo in range(0, 1 << 32, GPU_CHUNK):
            # the patterns lo .. lo+2^28-1 as int32 bits (a chunk never straddles 2^31)
            base = lo if lo < (1 << 31) else lo - (1 << 32)
            x = (idx + base).to(torch.int32).view(torch.float32)
            c = fq.e4m3_encode_f32(x)
            nan = torch.isnan(x)
            bad_nan = int(((c[nan] & 0x7F) != 0x7F).sum())
            assert bad_nan == 0, f"{bad_nan} NaN inputs near 0x{lo:08x} gave a non-NaN code"
            c[nan] = 0
            h = c.cpu().numpy()
            for s in range(0, GPU_CHUNK, SLICE):
                gpu_digests.append(hashlib.blake2b(h[s:s + SLICE].tobytes(), digest_size=16).digest())
            del x, c, nan
        oracle_digests = pending.get(timeout=3600)
    assert len(gpu_digests) == len(oracle_digests) == n_slices
    bad = [i for i in range(n_slices) if gpu_digests[i] != oracle_digests[i]]
    if bad:
        i = bad[0]
        lo = i * SLICE
        ref = worker.codes(lo, lo + SLICE)
        x = torch.from_numpy(np.arange(lo, lo + SLICE, dtype=np.uint64).astype(np.uint32).view(np.float32)).cuda()
        got = fq.e4m3_encode_f32(x).cpu().numpy()
        got[np.isnan(x.cpu().numpy())] = 0
        j = int(np.argwhere(got != ref)[0][0])
        raise AssertionError(f"{len(bad)} of {n_slices} slices differ; first at pattern 0x{lo + j:08x}: "
                             f"gpu 0x{got[j]:02x} oracle 0x{ref[j]:02x}")
    assert fq.device_error() == 0
