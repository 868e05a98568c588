"""GPU parity of the MoE expert grouped FP8 linear (fp8q_moe_grouped_linear).

Rows arrive grouped by expert (FP16 top-2 router and permutation are part of
the seeded input synthesis); offsets live on the device.  The oracle computes
every row with its expert's quantized weights and scales, and every row of
every output is compared, the full-size 16384-row up and down projections
included.  All device outputs sit inside guard-banded buffers (a seeded byte
pattern on each side, checked after the call), so a masked store at an expert
boundary that runs past the last row of the output is caught.
"""
import numpy as np
import pytest
import torch

from oracle import linear_ref, moe_ref, quant_rows
from fp8_quantized_generative_b200 import workloads as wl

from parity import Guards, assert_close_f16, assert_no_device_error, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import fp8_quantized_generative_b200 as m
    assert torch.cuda.is_available()
    return m


def run_gpu(fq, Xg, offsets, W):
    g = Guards()
    E, N, K = W.shape
    R = Xg.shape[0]
    Wq = g((E, N, K), torch.uint8, 0xFF, "Wq")
    s_w = g((E, N), torch.float32, float("nan"), "s_w")
    fq.quantize_weight_per_channel(W.cuda(), out=(Wq, s_w))
    Xq = g((R, K), torch.uint8, 0xFF, "Xq")
    s_x = g((R,), torch.float32, float("nan"), "s_x")
    fq.quantize_rows_dynamic(Xg.cuda(), out=(Xq, s_x))
    off = torch.from_numpy(np.asarray(offsets, dtype=np.int32)).cuda()
    # NaN-filled, guard-banded output: rows written past an expert group's end
    # land in a neighbour's rows (caught by the compare) or past the buffer
    # (caught by the guard bytes)
    Y = g((R, N), torch.float16, float("nan"), "Y")
    fq.moe_grouped_linear(Xq, s_x, off, Wq, s_w, out=Y)
    g.check(f"moe R={R} E={E} N={N} K={K}")
    return Y


def oracle_rows(Xg, offsets, W, rows):
    """Oracle output for the given rows only: each row with its own expert."""
    offsets = np.asarray(offsets, dtype=np.int64)
    E, N, K = W.shape
    expert_of = np.searchsorted(offsets, rows, side="right") - 1
    out = np.zeros((len(rows), N), np.float16)
    Xq, s_x = quant_rows(Xg.numpy()[rows])
    for e in np.unique(expert_of):
        sel = expert_of == e
        Wq, s_w = quant_rows(W[e].numpy())
        out[sel] = linear_ref(Xq[sel], s_x[sel], Wq, s_w)
    return out


@pytest.fixture(params=[0, 2], ids=["single", "pair"])
def family(request, fq):
    """Grouped kernel family: 0 = automatic (single CTA, 128-row blocks), 2 = CTA pairs (256-row blocks)."""
    fq.set_gemm_tuning(request.param, 0, 0)
    yield request.param
    fq.set_gemm_tuning(0, 0, 0)


def test_small_groups_full_compare(fq, family):
    E, N, K = 6, 264, 272
    counts = [0, 130, 1, 0, 300, 57]
    off = wl.offsets_from_counts(counts)
    R = int(off[-1])
    X = wl.random_f16((R, K), seed=11)
    W = wl.random_f16((E, N, K), seed=12, std=0.02)
    Y = run_gpu(fq, X, off, W)
    Wq, s_w = quant_rows(W.reshape(E * N, K).numpy())
    Xq, s_x = quant_rows(X.numpy())
    ref = moe_ref(Xq, s_x, off, Wq.reshape(E, N, K), s_w.reshape(E, N))
    assert_close_f16(to_np(Y), ref, "small groups")
    assert_no_device_error()


@pytest.mark.parametrize("counts", [
    [0, 0, 0, 513, 0],            # one expert holds every row
    [1, 1, 1, 1, 1, 1, 1, 1],     # single-row groups
    [128, 128, 256],              # exact tile multiples
    [700],                        # E = 1 behaves like a dense linear
    [255, 257, 0, 1, 512, 100],   # 256-row blocks split one row before / after the boundary
    # CTA-pair kernel: an expert's last 1..128 rows form an M = 128 pair tile
    # (64 rows per CTA), 129..255 an M = 256 tile; both sides of each edge
    [64, 65, 127, 128, 129, 191, 320, 383, 384, 385],
])
def test_adversarial_offsets(fq, family, counts):
    E, N, K = len(counts), 256, 256
    off = wl.offsets_from_counts(counts)
    R = int(off[-1])
    X = wl.random_f16((R, K), seed=R + E)
    W = wl.random_f16((E, N, K), seed=E + 1, std=0.02)
    Y = run_gpu(fq, X, off, W)
    assert_close_f16(to_np(Y), oracle_rows(X, off, W, np.arange(R)), f"counts={counts}")
    assert_no_device_error()


def test_bad_offsets_are_reported_and_nothing_written(fq, family):
    E, N, K = 3, 64, 128
    X = wl.random_f16((10, K), seed=1).cuda()
    Xq, s_x = fq.quantize_rows_dynamic(X)
    Wq = torch.zeros((E, N, K), dtype=torch.uint8, device="cuda")
    s_w = torch.ones((E, N), dtype=torch.float32, device="cuda")
    for bad in ([0, 6, 4, 10], [1, 4, 6, 10], [0, 4, 6, 9]):
        off = torch.tensor(bad, dtype=torch.int32, device="cuda")
        Y = torch.full((10, N), 7.0, dtype=torch.float16, device="cuda")
        fq.moe_grouped_linear(Xq, s_x, off, Wq, s_w, out=Y)
        flags = fq.device_error()
        assert flags == 0x8, hex(flags)
        assert torch.all(Y == 7.0)


@pytest.fixture(scope="module")
def moe_case():
    return wl.moe()


def test_moe_up_full(fq, family, moe_case):
    # every grouped row of the full-size up projection against the oracle
    m = moe_case
    Y = run_gpu(fq, m.X_perm, m.offsets, m.W_up)
    R = m.X_perm.shape[0]
    assert_close_f16(to_np(Y), oracle_rows(m.X_perm, m.offsets, m.W_up, np.arange(R)), "moe up")
    assert_no_device_error()


def test_moe_down_full(fq, family, moe_case):
    # Down projection on an independent seeded input of the up-output's shape.
    m = moe_case
    Xd = wl.random_f16((m.X_perm.shape[0], wl.MOE_F), seed=303)
    Y = run_gpu(fq, Xd, m.offsets, m.W_down)
    assert_close_f16(to_np(Y), oracle_rows(Xd, m.offsets, m.W_down, np.arange(Xd.shape[0])), "moe down")
    assert_no_device_error()
