"""GPU parity of the block-scaled MoE variant ('FP8量化在生成式推荐系统OneRec-V2中的
优化实践' §2.1: the MoE expert grouped GEMM quantized block-wise 128x128; §2.2:
block-aligned MoE quantization, activations per token).

* fp8q_quantize_weight_blockwise: codes and block scales bit-exact against
  oracle.quant_blocks, per expert (blocks never span experts);
* fp8q_moe_grouped_linear_blockscaled: FP16 outputs within the path's
  tolerance of oracle.moe_blockscaled_ref on ragged groups, adversarial
  offsets and the full MoE configuration (every row; guard-banded output).
"""
import numpy as np
import pytest
import torch

from oracle import linear_blockscaled_ref, moe_blockscaled_ref, quant_blocks, quant_rows
from fp8_quantized_generative_b200 import workloads as wl

from parity import Guards, assert_close_f16, assert_no_device_error, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import fp8_quantized_generative_b200 as m
    assert torch.cuda.is_available()
    return m


def oracle_blocks(W):
    """Per-expert oracle block quantization of W [E,N,K] (or [N,K])."""
    W3 = W.numpy() if W.dim() == 3 else W.numpy()[None]
    q = [quant_blocks(W3[e]) for e in range(W3.shape[0])]
    return np.stack([c for c, _ in q]), np.stack([s for _, s in q])


@pytest.mark.parametrize("E,N,K", [(1, 300, 272), (3, 200, 384), (2, 128, 128), (4, 136, 4112)])
def test_blockwise_quant_bit_exact(fq, E, N, K):
    W = wl.random_f16((E, N, K), seed=E * 100 + N + K, std=0.02)
    W[0, min(N - 1, 5), min(K - 1, 7)] = 0.5            # one block with a large maximum
    Wq, s = fq.quantize_weight_blockwise(W.cuda())
    torch.cuda.synchronize()
    ref_q, ref_s = oracle_blocks(W)
    got_q = to_np(Wq).reshape(ref_q.shape)
    if not np.array_equal(got_q, ref_q):
        bad = np.argwhere(got_q != ref_q)[0]
        raise AssertionError(f"code mismatch at {tuple(bad)}: gpu 0x{got_q[tuple(bad)]:02x} oracle 0x{ref_q[tuple(bad)]:02x}")
    np.testing.assert_array_equal(to_np(s).reshape(ref_s.shape).view(np.uint32), ref_s.view(np.uint32))
    assert_no_device_error()


def run_bs(fq, X, offsets, W):
    Wq, s_wb = fq.quantize_weight_blockwise(W.cuda())
    Xq, s_x = fq.quantize_rows_dynamic(X.cuda())
    off = torch.from_numpy(np.asarray(offsets, dtype=np.int32)).cuda()
    g = Guards()
    Y = g((X.shape[0], W.shape[1]), torch.float16, float("nan"), "Y")
    fq.moe_grouped_linear_blockscaled(Xq, s_x, off, Wq, s_wb, out=Y)
    g.check("block-scaled")
    return Y


def oracle_rows_bs(X, offsets, W, rows):
    offsets = np.asarray(offsets, dtype=np.int64)
    expert_of = np.searchsorted(offsets, rows, side="right") - 1
    out = np.zeros((len(rows), W.shape[1]), np.float16)
    Xq, s_x = quant_rows(X.numpy()[rows])
    for e in np.unique(expert_of):
        sel = expert_of == e
        Wq, s_wb = quant_blocks(W[e].numpy())
        out[sel] = linear_blockscaled_ref(Xq[sel], s_x[sel], Wq, s_wb)
    return out


def test_small_groups_full_compare(fq):
    E, N, K = 5, 264, 272
    counts = [0, 130, 1, 300, 57]
    off = wl.offsets_from_counts(counts)
    R = int(off[-1])
    X = wl.random_f16((R, K), seed=41)
    W = wl.random_f16((E, N, K), seed=42, std=0.02)
    W[1, :, 130:140] *= 20                               # block scales that differ along K
    Y = run_bs(fq, X, off, W)
    Xq, s_x = quant_rows(X.numpy())
    Wq, s_wb = oracle_blocks(W)
    assert_close_f16(to_np(Y), moe_blockscaled_ref(Xq, s_x, off, Wq, s_wb), "block-scaled small groups")
    assert_no_device_error()


@pytest.mark.parametrize("counts", [
    [0, 0, 513, 0],
    [1, 1, 1, 1, 1],
    [128, 129, 255, 256, 257],
    [700],
])
def test_adversarial_offsets(fq, counts):
    E, N, K = len(counts), 256, 512
    off = wl.offsets_from_counts(counts)
    R = int(off[-1])
    X = wl.random_f16((R, K), seed=R + 3 * E)
    W = wl.random_f16((E, N, K), seed=E + 17, std=0.02)
    W[:, :, 256:384] *= 8
    Y = run_bs(fq, X, off, W)
    assert_close_f16(to_np(Y), oracle_rows_bs(X, off, W, np.arange(R)), f"counts={counts}")
    assert_no_device_error()


def test_bad_offsets_are_reported_and_nothing_written(fq):
    E, N, K = 3, 128, 128
    X = wl.random_f16((10, K), seed=1).cuda()
    Xq, s_x = fq.quantize_rows_dynamic(X)
    Wq, s_wb = fq.quantize_weight_blockwise(wl.random_f16((E, N, K), seed=2, std=0.02).cuda())
    for bad in ([0, 6, 4, 10], [1, 4, 6, 10], [0, 4, 6, 9]):
        off = torch.tensor(bad, dtype=torch.int32, device="cuda")
        Y = torch.full((10, N), 7.0, dtype=torch.float16, device="cuda")
        fq.moe_grouped_linear_blockscaled(Xq, s_x, off, Wq, s_wb, out=Y)
        assert fq.device_error() == 0x8
        assert torch.all(Y == 7.0)


@pytest.fixture(scope="module")
def moe_case():
    return wl.moe()


def test_moe_up_blockscaled(fq, moe_case):
    m = moe_case
    Y = run_bs(fq, m.X_perm, m.offsets, m.W_up)
    rows = np.arange(m.X_perm.shape[0])            # every grouped row
    assert_close_f16(to_np(Y), oracle_rows_bs(m.X_perm, m.offsets, m.W_up, rows), "block-scaled moe up")
    assert_no_device_error()


def test_moe_down_blockscaled(fq, moe_case):
    m = moe_case
    Xd = wl.random_f16((m.X_perm.shape[0], wl.MOE_F), seed=304)
    Y = run_bs(fq, Xd, m.offsets, m.W_down)
    rows = np.arange(Xd.shape[0])                  # every grouped row
    assert_close_f16(to_np(Y), oracle_rows_bs(Xd, m.offsets, m.W_down, rows), "block-scaled moe down")
    assert_no_device_error()
