"""Failure detection without a GPU fault: a device wait that nothing will
satisfy must give up after its limit, report through the device error word,
and leave the CUDA context usable."""
import numpy as np
import pytest
import torch

from fp8_quantized_generative_b200 import _lib
from fp8_quantized_generative_b200 import workloads as wl
from oracle import linear_ref, quant_rows

from parity import assert_close_f16, to_np

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    import fp8_quantized_generative_b200 as fq
    assert fq.device_error() == 0
    stream = torch.cuda.current_stream().cuda_stream
    assert _lib.fp8q_selftest_wait_timeout(2000, stream) == _lib.FP8Q_OK     # 2 ms limit
    st, flags = _lib.fp8q_device_error(stream)
    assert st == _lib.FP8Q_ERR_TIMEOUT
    assert flags == _lib.DEVERR_TIMEOUT_SELFTEST
    assert fq.device_error() == 0                                            # read clears it
    # the context still runs the real path
    lin = wl.tiny()
    Wq, s_w = fq.quantize_weight_per_channel(lin.W.cuda())
    Xq, s_x = fq.quantize_rows_dynamic(lin.X.cuda())
    Y = fq.linear(Xq, s_x, Wq, s_w)
    rq, rs = quant_rows(lin.X.numpy())
    wq, ws = quant_rows(lin.W.numpy())
    assert_close_f16(to_np(Y), linear_ref(rq, rs, wq, ws), "after timeout")
    assert fq.device_error() == 0

