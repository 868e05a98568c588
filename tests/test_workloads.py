"""Checks of the seeded synthetic inputs and the FP16 top-2 router (harness only)."""
import numpy as np
import pytest
import torch

from fp8_quantized_generative_b200 import workloads as wl


def test_router_brute_force_with_ties():
    rng = np.random.default_rng(0)
    for trial in range(20):
        T, E = int(rng.integers(1, 40)), int(rng.integers(2, 9))
        # few distinct values -> many exact ties
        logits = rng.integers(-2, 3, size=(T, E)).astype(np.float16)
        got = wl.route_top2(logits)
        for t in range(T):
            order = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))
            assert list(got[t]) == order[:2]


def test_grouping_brute_force():
    rng = np.random.default_rng(1)
    T, E = 50, 7
    logits = rng.standard_normal((T, E)).astype(np.float16)
    ex = wl.route_top2(logits)
    tok, off = wl.group_by_expert(ex, E)
    assert off[0] == 0 and off[-1] == 2 * T and np.all(np.diff(off) >= 0)
    rows = []
    for e in range(E):
        for t in range(T):
            if e in ex[t]:
                rows.append(t)
    assert list(tok) == rows
    for e in range(E):
        seg = tok[off[e]:off[e + 1]]
        assert all(e in ex[t] for t in seg)


def test_moe_workload_structure():
    m = wl.moe(T=512, with_weights=False)
    assert m.offsets.dtype == np.int32 and m.offsets.shape == (wl.MOE_E + 1,)
    assert m.offsets[-1] == 2 * 512
    # each token appears exactly twice, in two distinct experts
    counts = np.bincount(m.token_of_row, minlength=512)
    assert np.all(counts == 2)
    assert torch.equal(m.X_perm, m.X[torch.from_numpy(m.token_of_row)])


def test_inputs_are_deterministic_and_shaped():
    a, b = wl.tiny(), wl.tiny()
    assert torch.equal(a.X, b.X) and torch.equal(a.W, b.W)
    assert a.X.shape == (32, 256) and a.W.shape == (256, 256) and a.X.dtype == torch.float16
    w_std = a.W.float().std().item()
    assert 0.017 < w_std < 0.023


def test_qkv_outlier_channels():
    lin = wl.qkv(m=256)
    col_max = lin.X.float().abs().amax(dim=0)
    big = (col_max > 20).sum().item()
    assert big == 20                       # 1% of 2048 channels scaled by 50
    assert lin.X.float().abs().max().item() < 400


def test_sweep_lognormal_signs():
    x = wl.sweep_x(64).float()
    assert x.shape == (64, 4096)
    assert 0.45 < (x > 0).float().mean().item() < 0.55
    lm = x.abs().log()
    assert abs(lm.mean().item()) < 0.05 and 0.95 < lm.std().item() < 1.05


def test_token_rows_inverts_the_grouping():
    rng = np.random.default_rng(5)
    T, E = 37, 6
    logits = rng.standard_normal((T, E)).astype(np.float16)
    row_token, _ = wl.group_by_expert(wl.route_top2(logits), E)
    tr = wl.token_rows(row_token, T)
    assert tr.shape == (T, 2) and tr.dtype == np.int32
    # every grouped row appears exactly once, under its own token
    flat = tr.reshape(-1)
    assert np.array_equal(np.sort(flat[flat >= 0]), np.arange(len(row_token)))
    for t in range(T):
        for r in tr[t]:
            assert r == -1 or row_token[r] == t
    # a token with fewer rows than topk is padded with -1
    tr1 = wl.token_rows(np.array([2, 0, 2]), 4)
    assert tr1.tolist() == [[1, -1], [-1, -1], [0, 2], [-1, -1]]
    with pytest.raises(ValueError):
        wl.token_rows(np.array([1, 1, 1]), 2)


def test_gate_weights_and_row_weights():
    # softmax over each token's selected logits, highest logit first; the row
    # weights follow the grouped-row order of group_by_expert
    logits = np.array([[0.0, 1.0, -1.0, 2.0], [3.0, 3.0, 0.0, -2.0]], np.float16)
    experts = wl.route_top2(logits)
    assert experts.tolist() == [[3, 1], [0, 1]]
    g = wl.gate_weights(logits, experts)
    e = 1.0 / (1.0 + np.exp(-1.0))                 # softmax of (2, 1): e^2 / (e^2 + e^1)
    np.testing.assert_allclose(g[0], [e, 1 - e], rtol=1e-6)
    np.testing.assert_allclose(g[1], [0.5, 0.5], rtol=1e-6)     # equal logits
    assert g.dtype == np.float32 and np.allclose(g.sum(axis=1), 1.0)
    row_token, offsets = wl.group_by_expert(experts, 4)
    rw = wl.row_weights(g, experts)
    # grouped rows: expert 0: token 1; expert 1: tokens 0, 1; expert 3: token 0
    assert row_token.tolist() == [1, 0, 1, 0] and list(offsets) == [0, 1, 3, 3, 4]
    np.testing.assert_allclose(rw, [g[1, 0], g[0, 1], g[1, 1], g[0, 0]], rtol=0)
