"""The parity tests' guard bands, checked on the CPU: they catch a write one
byte past either end of a tensor, and only then."""
import pytest
import torch

from parity import Guarded


def test_guard_passes_when_only_the_interior_is_written():
    g = Guarded((5, 7), torch.float16, fill=float("nan"), device="cpu")
    g.t.fill_(1.0)
    g.check("interior")


@pytest.mark.parametrize("where", ["before", "after"])
def test_guard_catches_a_one_byte_overrun(where):
    g = Guarded((3, 16), torch.uint8, fill=0, device="cpu")
    i = g.pad - 1 if where == "before" else g.pad + g.nbytes
    g.buf[i] = g.buf[i] ^ 0xFF
    with pytest.raises(AssertionError, match=where):
        g.check("planted overrun")


def test_guarded_interior_is_16_byte_aligned_and_contiguous():
    g = Guarded((33, 24), torch.float32, device="cpu")
    assert g.t.is_contiguous() and g.t.data_ptr() % 16 == 0 and tuple(g.t.shape) == (33, 24)
