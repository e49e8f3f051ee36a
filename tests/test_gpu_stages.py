"""Stage-by-stage parity of the CUDA path against the fp64 oracle, through the
C ABI. Integer results (indices, counts, offsets, permutation, statistics)
must be bit-exact; floating results within the stated tolerances."""
import math

import numpy as np
import pytest
import torch

import oracle
from parity import (BF16_Y_TOL, F32_Y_TOL, W_TOL, rel_max_err, stats_equal, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    from _lib import build_and_import
    return build_and_import()


def _i32(n):
    return torch.empty(n, dtype=torch.int32, device="cuda")


def _tie_logits(rng, T, E):
    vals = np.array([-1.5, -0.5, -0.0, 0.0, 0.25, 0.25, 1.0, 2.0], dtype=np.float32)
    return rng.choice(vals, size=(T, E)).astype(np.float32)


# ------------------------------------------------------------- selection ---
@pytest.mark.parametrize("T,E,K,ties,bias", [
    (1, 1, 1, False, False), (37, 7, 3, True, True), (64, 16, 2, True, False),
    (513, 128, 8, False, True), (300, 128, 8, True, True), (200, 256, 8, False, True),
    (129, 512, 16, True, True), (50, 16, 16, False, True), (1000, 64, 1, True, False)])
def test_topk_from_logits_bit_exact(M, T, E, K, ties, bias):
    rng = np.random.default_rng(T * 31 + E)
    logits = _tie_logits(rng, T, E) if ties else rng.normal(size=(T, E)).astype(np.float32)
    b = rng.uniform(-0.5, 0.5, size=E).astype(np.float32) if bias else None
    if ties and bias:
        b = rng.choice(np.array([-0.25, 0.0, -0.0, 0.25], np.float32), size=E)
    d = M.make_desc(T, 256, E, K, 256, 0, M.MOE_F32)
    lg = torch.from_numpy(logits).cuda()
    bd = torch.from_numpy(b).cuda() if b is not None else None
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    M.moe_topk_from_logits(d, lg, bd, idx, w)
    ref_idx, ref_w, _ = oracle.select_topk(logits.astype(np.float64), b, K)
    assert (to_np(idx) == ref_idx).all()
    assert np.max(np.abs(to_np(w) - ref_w)) <= W_TOL


# -------------------------------------------------------------- dispatch ---
@pytest.mark.parametrize("T,E,K,skew", [(1, 1, 1, 0), (5, 4, 4, 0), (64, 16, 2, 0), (333, 128, 8, 0.8),
                                        (3000, 128, 8, 1.0), (700, 256, 8, 1.5), (4096, 8, 2, 0),
                                        (17, 512, 16, 0.5), (20000, 128, 8, 0.4)])
def test_dispatch_bit_exact(M, T, E, K, skew):
    rng = np.random.default_rng(T + E * 7)
    idx_np, _, _ = oracle.select_topk(rng.normal(size=(T, E)), -skew * np.log(np.arange(E) + 1.0), K)
    d = M.make_desc(T, 128, E, K, 128, 0, M.MOE_BF16)
    ws = M.alloc_workspace(d)
    idx = torch.from_numpy(idx_np).cuda()
    counts, offsets, perm, inv = _i32(E), _i32(E + 1), _i32(T * K), _i32(T * K)
    M.moe_dispatch(d, idx, counts, offsets, perm, inv, ws)
    rc, ro, rp, ri = oracle.dispatch(idx_np, E)
    assert (to_np(counts) == rc).all() and (to_np(offsets) == ro).all()
    assert (to_np(perm) == rp).all() and (to_np(inv) == ri).all()
    assert M.moe_check_status(ws) == 0


def test_dispatch_empty_batch(M):
    d = M.make_desc(0, 128, 8, 2, 128, 0, M.MOE_BF16)
    ws = M.alloc_workspace(d)
    counts, offsets = _i32(8).fill_(-1), _i32(9).fill_(-1)
    M.moe_dispatch(d, None, counts, offsets, None, None, ws)
    assert (to_np(counts) == 0).all() and (to_np(offsets) == 0).all()


def test_dispatch_reports_out_of_range_index(M):
    d = M.make_desc(4, 128, 8, 2, 128, 0, M.MOE_BF16)
    ws = M.alloc_workspace(d)
    idx = torch.tensor([[0, 1], [2, 9], [3, 4], [5, 6]], dtype=torch.int32, device="cuda")
    M.moe_dispatch(d, idx, _i32(8), _i32(9), _i32(8), _i32(8), ws)
    assert M.moe_check_status(ws) == 1          # MOE_ERR_INVALID_ARG, then cleared
    assert M.moe_check_status(ws) == 0


# ------------------------------------------------------------ grouped FFN ---
@pytest.mark.parametrize("dtype,T,H,E,K,D,Ds", [
    ("f32", 64, 256, 16, 2, 512, 0), ("f32", 33, 64, 5, 3, 96, 32),
    ("bf16", 40, 256, 8, 2, 384, 0), ("bf16", 77, 256, 16, 4, 128, 256)])
def test_grouped_ffn_matches_oracle(M, dtype, T, H, E, K, D, Ds):
    rng = np.random.default_rng(T + H + D)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    q = lambda a: torch.from_numpy(a.astype(np.float32)).to(tdt)
    x = q(rng.normal(size=(T, H)))
    w1 = q(rng.normal(size=(E, D, H)) / math.sqrt(H))
    w2 = q(rng.normal(size=(E, H, D)) / math.sqrt(D))
    ws1 = q(rng.normal(size=(Ds, H)) / math.sqrt(H)) if Ds else None
    ws2 = q(rng.normal(size=(H, Ds)) / math.sqrt(Ds)) if Ds else None
    idx_np, _, _ = oracle.select_topk(rng.normal(size=(T, E)), -0.7 * np.log(np.arange(E) + 1.0), K)
    _, off_np, perm_np, _ = oracle.dispatch(idx_np, E)
    d = M.make_desc(T, H, E, K, D, Ds, M.MOE_F32 if dtype == "f32" else M.MOE_BF16)
    ws = M.alloc_workspace(d)
    dev = lambda t: t.cuda() if t is not None else None
    y_rows = torch.empty((T * K, H), dtype=torch.float32, device="cuda")   # expert outputs: fp32
    y_sh = torch.empty((T, H), dtype=torch.float32, device="cuda") if Ds else None
    M.moe_grouped_ffn(d, dev(x), torch.from_numpy(perm_np).cuda(), torch.from_numpy(off_np).cuda(),
                      dev(w1), dev(w2), dev(ws1), dev(ws2), y_rows, y_sh, ws)
    f64 = lambda t: t.double().numpy() if t is not None else None
    ref_rows, ref_sh = oracle.grouped_ffn(f64(x), perm_np, off_np, K, f64(w1), f64(w2), f64(ws1), f64(ws2))
    tol = F32_Y_TOL if dtype == "f32" else BF16_Y_TOL
    assert rel_max_err(to_np(y_rows), ref_rows) <= tol
    if Ds:
        assert rel_max_err(to_np(y_sh), ref_sh) <= tol


# --------------------------------------------------------------- combine ---
@pytest.mark.parametrize("dtype,T,H,K,shared", [("f32", 64, 256, 2, False), ("f32", 9, 64, 5, True),
                                                ("bf16", 300, 4096, 8, True), ("bf16", 1, 128, 1, False)])
def test_combine_matches_oracle(M, dtype, T, H, K, shared):
    rng = np.random.default_rng(T * H + K)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    rows = torch.from_numpy(rng.normal(size=(T * K, H)).astype(np.float32))   # fp32 expert outputs
    w = rng.random(size=(T, K)).astype(np.float32)
    w /= w.sum(1, keepdims=True)
    perm = rng.permutation(T * K).astype(np.int32)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(T * K, dtype=np.int32)
    sh = torch.from_numpy(rng.normal(size=(T, H)).astype(np.float32)) if shared else None
    d = M.make_desc(T, H, 8, K, 128, 128 if shared else 0, M.MOE_F32 if dtype == "f32" else M.MOE_BF16)
    y = torch.empty((T, H), dtype=tdt, device="cuda")
    M.moe_combine(d, rows.cuda(), torch.from_numpy(w).cuda(), torch.from_numpy(inv).cuda(),
                  sh.cuda() if shared else None, y)
    ref = oracle.combine(rows.double().numpy(), w.astype(np.float64), inv,
                         sh.double().numpy() if shared else None)
    if dtype == "f32":
        assert rel_max_err(to_np(y), ref) <= F32_Y_TOL
    else:   # one rounding of the fp32 sum to bf16: |err| <= 2^-8 |y| (+ fp32 summation noise)
        rms = np.sqrt(np.mean(ref ** 2))
        assert (np.abs(to_np(y) - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * rms).all()


# ------------------------------------------------------------------ stats ---
@pytest.mark.parametrize("E,T,K", [(16, 64, 2), (128, 1, 8), (128, 16384, 8), (256, 256, 8), (8, 4096, 2),
                                   (512, 100, 16), (1, 5, 1)])
def test_expert_stats_bit_exact(M, E, T, K):
    rng = np.random.default_rng(E + T)
    for trial in range(4):
        p = rng.dirichlet(np.full(E, 0.3 if trial % 2 else 5.0))
        counts_np = rng.multinomial(T * K, p).astype(np.int32)
        if trial == 3:
            counts_np[:] = (T * K) // E
            counts_np[0] += T * K - counts_np.sum()
        d = M.make_desc(T, 128, E, K, 128, 0, M.MOE_BF16)
        ws = M.alloc_workspace(d)
        mask = torch.empty(E, dtype=torch.uint8, device="cuda")
        got = M.moe_expert_stats(d, torch.from_numpy(counts_np).cuda(), mask, ws)
        want = oracle.load_stats(counts_np, T, K)
        stats_equal(got, want)
        assert (to_np(mask) == want["straggler_mask"]).all()


def test_expert_stats_golden_cases(M):
    import json, os
    cases = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "load_stats_cases.json")))
    for case in cases["stats"]:
        if "counts" in case:
            counts_np = np.array(case["counts"], dtype=np.int32)
        else:
            counts_np = np.zeros(case["E"], dtype=np.int32)
            counts_np[case["hot"]] = 1
        E = counts_np.size
        d = M.make_desc(case["T"], 128, E, case["K"], 128, 0, M.MOE_BF16)
        ws = M.alloc_workspace(d)
        got = M.moe_expert_stats(d, torch.from_numpy(counts_np).cuda(), None, ws)
        for key in ("capacity", "max_load", "min_load", "overflow", "num_stragglers"):
            assert got[key] == case[key], key
        assert got["overflow_rate"] == pytest.approx(case["overflow_rate"], abs=1e-15)
    for case in cases["gini"]:
        c = np.array(case["counts"], dtype=np.int32)
        d = M.make_desc(max(1, int(c.sum())), 128, c.size, 1, 128, 0, M.MOE_BF16)
        ws = M.alloc_workspace(d)
        got = M.moe_expert_stats(d, torch.from_numpy(c).cuda(), None, ws)
        want = case["gini"] if "gini" in case else case["gini_num"] / case["gini_den"]
        assert got["gini"] == pytest.approx(want, abs=1e-15)
