"""Dynamic expert bias update ("Kimi K3 专家路由不均衡诊断" §四) on the GPU
against the oracle: the fp32 bias must match bit for bit, alone and inside
a closed routing loop (select -> dispatch -> counts -> update)."""
import numpy as np
import pytest
import torch

import oracle
from parity import to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    from _lib import build_and_import
    return build_and_import()


def _bits(a):
    return np.asarray(a, dtype=np.float32).view(np.int32)


@pytest.mark.parametrize("E,T,K,gamma,kind", [
    (1, 4, 1, 0.01, "uniform"), (6, 16, 3, 0.125, "hand"), (64, 512, 6, 1e-3, "zipf"),
    (128, 4096, 8, 1e-3, "zipf"), (512, 777, 16, 0.05, "sparse"), (256, 100, 8, 0.0, "zipf"),
    (160, 2048, 6, 3e-4, "large_bias")])
def test_bias_update_bit_exact(M, E, T, K, gamma, kind):
    rng = np.random.default_rng(E * 13 + T)
    TK = T * K
    if kind == "hand":
        counts = np.array([30, 0, 5, 10, 0, 11], np.int32)
    elif kind == "uniform":
        counts = np.full(E, TK // E, np.int32)
    elif kind == "sparse":          # many idle experts, a few hot ones
        counts = np.zeros(E, np.int32)
        hot = rng.choice(E, size=8, replace=False)
        counts[hot] = rng.multinomial(TK, np.full(8, 1 / 8))
    else:
        p = 1.0 / np.arange(1, E + 1) ** 1.1
        counts = rng.multinomial(TK, p / p.sum()).astype(np.int32)
    scale = 1e4 if kind == "large_bias" else 0.5
    bias = rng.uniform(-scale, scale, size=E).astype(np.float32)
    bias[: min(E, 3)] = np.array([0.0, -0.0, 1e-8], np.float32)[: min(E, 3)]
    d = M.make_desc(T, 128, E, K, 128, 0, M.MOE_BF16)
    b_dev = torch.from_numpy(bias.copy()).cuda()
    M.moe_bias_update(d, torch.from_numpy(counts).cuda(), b_dev, gamma)
    ref = oracle.bias_update(bias, counts, T, K, gamma)
    assert (_bits(to_np(b_dev)) == _bits(ref)).all()


def test_bias_update_closed_loop(M):
    """A skewed router driven by its own bias: every step's counts and bias
    match the oracle exactly, and the load evens out."""
    T, E, K, gamma, steps = 512, 64, 6, 0.02, 40
    rng = np.random.default_rng(2024)
    skew = (-0.6 * np.log(np.arange(E) + 1.0)).astype(np.float32)
    d = M.make_desc(T, 256, E, K, 256, 0, M.MOE_F32)
    ws = M.alloc_workspace(d)
    bias = np.zeros(E, np.float32)
    b_dev = torch.zeros(E, dtype=torch.float32, device="cuda")
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * K, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * K, dtype=torch.int32, device="cuda")
    gini = []
    for _ in range(steps):
        logits = (rng.normal(size=(T, E)).astype(np.float32) + skew).astype(np.float32)
        M.moe_topk_from_logits(d, torch.from_numpy(logits).cuda(), b_dev, idx, w)
        M.moe_dispatch(d, idx, counts, offsets, perm, inv, ws)
        M.moe_bias_update(d, counts, b_dev, gamma)
        ref_idx, _, _ = oracle.select_topk(logits.astype(np.float64), bias, K)
        ref_counts = oracle.expert_counts(ref_idx, E)
        bias = oracle.bias_update(bias, ref_counts, T, K, gamma)
        assert (to_np(counts) == ref_counts).all()
        assert (_bits(to_np(b_dev)) == _bits(bias)).all()
        gini.append(oracle.gini_exact(ref_counts))
    assert M.moe_check_status(ws) == 0
    assert np.mean(gini[-5:]) < 0.7 * np.mean(gini[:3])
