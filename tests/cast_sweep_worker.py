"""Worker of the exhaustive device-cast test (test_zy_cast_sweep.py), kept in
a module of its own so that the spawned pool processes import only NumPy and
the oracle, not torch.

digest(lo, hi): the oracle's E4M3 codes of every fp32 bit pattern in
[lo, hi), with the codes of NaN inputs (outside the contract) set to 0,
reduced to a BLAKE2b digest.  The GPU side builds the same digest from the
device cast, so a single differing code changes it.
"""
import hashlib

import numpy as np

from oracle import e4m3_encode


def codes(lo: int, hi: int) -> np.ndarray:
    bits = np.arange(lo, hi, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    c = e4m3_encode(v)
    c[np.isnan(v)] = 0
    return c


def digest(lo: int, hi: int) -> bytes:
    return hashlib.blake2b(codes(lo, hi).tobytes(), digest_size=16).digest()
