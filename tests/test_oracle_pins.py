"""Pins for the fp64 oracle: it is checked against things other than itself.

Each test ties one oracle step to a closed form, a brute-force enumeration,
an independent library routine (torch float64 layers, scipy softmax), an
invariant the pages' definitions imply, or hand-derived values stored under
``tests/golden/`` with their derivation.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.special import softmax as sp_softmax

import oracle
import moe_inputs as mi

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _tie_logits(rng, T, E):
    """Logits from a small value set so that ties (and -0.0 / +0.0) are frequent."""
    vals = np.array([-1.5, -0.5, -0.0, 0.0, 0.25, 0.25, 1.0, 2.0], dtype=np.float64)
    return rng.choice(vals, size=(T, E))


# ----------------------------------------------------------------- top-K ---
def _brute_force_set(s_row, K):
    """The unique K-subset whose every member beats every non-member under
    (score descending, expert index ascending)."""
    E = len(s_row)
    found = []
    for sub in itertools.combinations(range(E), K):
        inside = set(sub)
        ok = all((s_row[i] > s_row[j]) or (s_row[i] == s_row[j] and i < j)
                 for i in inside for j in range(E) if j not in inside)
        if ok:
            found.append(inside)
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_brute_force_enumeration(seed):
    rng = _rng(seed)
    for E in range(1, 9):
        for K in range(1, min(E, 4) + 1):
            logits = _tie_logits(rng, 12, E) if seed % 2 == 0 else rng.normal(size=(12, E))
            bias = None if seed % 3 == 0 else rng.choice([-0.5, 0.0, 0.5], size=E)
            idx, w, s = oracle.select_topk(logits, bias, K)
            for t in range(logits.shape[0]):
                assert set(idx[t].tolist()) == _brute_force_set(s[t].astype(np.float64), K)
                # slots: descending score, ties by ascending expert index
                keys = [(-float(s[t, e]), int(e)) for e in idx[t]]
                assert keys == sorted(keys)


def test_selection_is_decided_in_fp32():
    # l = [1, 1], B = [0, 2^-25]: in fp32 1 + 2^-25 rounds to 1 -> tie -> expert 0;
    # an fp64 decision would pick expert 1.
    logits = np.array([[1.0, 1.0]])
    idx, _, s = oracle.select_topk(logits, np.array([0.0, 2.0 ** -25]), 1)
    assert s[0, 0] == s[0, 1] and idx[0, 0] == 0
    # and a gap that survives fp32 rounding is honoured
    idx, _, _ = oracle.select_topk(logits, np.array([0.0, 2.0 ** -22]), 1)
    assert idx[0, 0] == 1


def test_negative_and_positive_zero_tie_to_lower_index():
    logits = np.array([[0.0, -0.0, -1.0], [-0.0, 0.0, -1.0]])
    idx, w, _ = oracle.select_topk(logits, None, 1)
    assert idx[:, 0].tolist() == [0, 0]
    idx, w, _ = oracle.select_topk(logits, None, 2)
    assert idx.tolist() == [[0, 1], [0, 1]]
    assert np.allclose(w, 0.5, atol=0, rtol=0)


def test_K_equals_E_gives_full_softmax():
    rng = _rng(11)
    for E in (1, 2, 5, 16):
        logits = rng.normal(size=(20, E)) * 3
        bias = rng.normal(size=E)
        idx, w, s = oracle.select_topk(logits, bias, E)
        full = sp_softmax(s.astype(np.float64), axis=1)
        np.testing.assert_allclose(w, np.take_along_axis(full, idx, 1), rtol=1e-13, atol=1e-15)


def test_weights_sum_to_one_and_ratio_is_exp_gap():
    rng = _rng(12)
    logits = rng.normal(size=(200, 64)) * 2
    bias = rng.uniform(-0.5, 0.5, size=64)
    idx, w, s = oracle.select_topk(logits, bias, 8)
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-12, rtol=0)
    ss = np.take_along_axis(s, idx, 1).astype(np.float64)
    np.testing.assert_allclose(w[:, 1:] / w[:, :1], np.exp(ss[:, 1:] - ss[:, :1]), rtol=1e-12)
    assert (np.diff(w, axis=1) <= 0).all()


def test_E1_or_K1_weight_is_exactly_one():
    rng = _rng(13)
    _, w, _ = oracle.select_topk(rng.normal(size=(9, 1)), None, 1)
    assert (w == 1.0).all()
    _, w, _ = oracle.select_topk(rng.normal(size=(9, 7)), rng.normal(size=7), 1)
    assert (w == 1.0).all()


def test_router_matches_page_pipeline_in_torch_fp64():
    """The router code on the Kimi K3 All-to-All page (gate Linear without bias,
    softmax, topk, renormalise), run with torch float64 layers, selects the
    same experts with the same weights when no scores are tied."""
    rng = _rng(14)
    T, H, E, K = 64, 48, 32, 8
    x = rng.normal(size=(T, H))
    wr = rng.normal(size=(E, H)) / math.sqrt(H)
    bias = rng.uniform(-0.5, 0.5, size=E)
    gate = torch.nn.Linear(H, E, bias=False).double()
    with torch.no_grad():
        gate.weight.copy_(torch.from_numpy(wr))
        lt = gate(torch.from_numpy(x))
    scores = torch.softmax(lt + torch.from_numpy(bias), dim=-1)
    tw, ti = torch.topk(scores, K, dim=-1)
    tw = tw / tw.sum(dim=-1, keepdim=True)
    idx, w, _ = oracle.select_topk(oracle.router_logits(x, wr), bias, K)
    np.testing.assert_allclose(oracle.router_logits(x, wr), lt.numpy(), rtol=1e-12, atol=1e-12)
    assert (idx == ti.numpy()).all()
    # weights differ only by the fp32 rounding of the scores the decision uses
    np.testing.assert_allclose(w, tw.numpy(), rtol=0, atol=2e-6)


# -------------------------------------------------------------- dispatch ---
def _check_dispatch_invariants(idx, E, counts, off, perm, inv):
    T, K = idx.shape
    flat = idx.reshape(-1)
    assert counts.sum() == T * K
    assert off[0] == 0 and off[-1] == T * K and (np.diff(off) == counts).all()
    assert (np.diff(off) >= 0).all()
    assert sorted(perm.tolist()) == list(range(T * K))             # bijection
    assert (inv[perm] == np.arange(T * K)).all()                    # inv o perm = id
    for e in range(E):
        seg = perm[off[e]:off[e + 1]]
        assert (flat[seg] == e).all()                                # right segment
        assert (np.diff(seg) > 0).all()                              # ascending token


def _brute_force_dispatch(idx, E):
    T, K = idx.shape
    lists = [[] for _ in range(E)]
    for t in range(T):
        for k in range(K):
            lists[int(idx[t, k])].append(t * K + k)
    counts = [len(l) for l in lists]
    perm = [c for l in lists for c in l]
    return counts, perm


@pytest.mark.parametrize("T,E,K", [(1, 1, 1), (5, 4, 4), (37, 8, 2), (64, 16, 2), (50, 128, 8), (3, 256, 8)])
def test_dispatch_invariants_and_brute_force(T, E, K):
    rng = _rng(T * 7 + E)
    logits = rng.normal(size=(T, E))
    bias = -0.9 * np.log(np.arange(E) + 1.0)          # skew: many idle experts
    idx, _, _ = oracle.select_topk(logits, bias, K)
    counts, off, perm, inv = oracle.dispatch(idx, E)
    _check_dispatch_invariants(idx, E, counts, off, perm, inv)
    bc, bp = _brute_force_dispatch(idx, E)
    assert counts.tolist() == bc and perm.tolist() == bp


def test_dispatch_empty_batch():
    idx = np.zeros((0, 2), dtype=np.int32)
    counts, off, perm, inv = oracle.dispatch(idx, 4)
    assert counts.tolist() == [0] * 4 and off.tolist() == [0] * 5
    assert perm.size == 0 and inv.size == 0


# ------------------------------------------------------------------- FFN ---
def test_gelu_closed_forms_and_torch():
    phi1 = 0.5 * (1 + math.erf(1 / math.sqrt(2)))
    assert oracle.gelu_erf(np.array([0.0]))[0] == 0.0
    assert abs(oracle.gelu_erf(np.array([1.0]))[0] - phi1) < 1e-15
    assert abs(oracle.gelu_erf(np.array([-1.0]))[0] + (1 - phi1)) < 1e-15
    z = np.linspace(-9, 9, 1001)
    np.testing.assert_allclose(oracle.gelu_erf(z) - oracle.gelu_erf(-z), z, atol=1e-14)
    ref = F.gelu(torch.from_numpy(z), approximate="none").numpy()
    np.testing.assert_allclose(oracle.gelu_erf(z), ref, rtol=1e-14, atol=1e-15)
    assert oracle.gelu_erf(np.array([40.0]))[0] == 40.0 and oracle.gelu_erf(np.array([-40.0]))[0] == 0


def _torch_ffn(x, w1, w2):
    with torch.no_grad():
        h = F.gelu(F.linear(torch.from_numpy(x), torch.from_numpy(w1)), approximate="none")
        return F.linear(h, torch.from_numpy(w2)).numpy()


def _rand_layer(rng, T, H, E, D, Ds=0):
    x = rng.normal(size=(T, H))
    wr = rng.normal(size=(E, H)) / math.sqrt(H)
    w1 = rng.normal(size=(E, D, H)) / math.sqrt(H)
    w2 = rng.normal(size=(E, H, D)) / math.sqrt(D)
    ws1 = rng.normal(size=(Ds, H)) / math.sqrt(H) if Ds else None
    ws2 = rng.normal(size=(H, Ds)) / math.sqrt(Ds) if Ds else None
    return x, wr, w1, w2, ws1, ws2


def test_E1_K1_reduces_to_dense_ffn():
    rng = _rng(21)
    x, wr, w1, w2, ws1, ws2 = _rand_layer(rng, 33, 40, 1, 72, Ds=24)
    out = oracle.moe_layer_forward(x, wr, None, w1, w2, None, None, 1)
    np.testing.assert_allclose(out["y"], _torch_ffn(x, w1[0], w2[0]), rtol=1e-12, atol=1e-12)
    out = oracle.moe_layer_forward(x, wr, None, w1, w2, ws1, ws2, 1)
    np.testing.assert_allclose(out["y"], _torch_ffn(x, w1[0], w2[0]) + _torch_ffn(x, ws1, ws2),
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("K", [1, 2, 3, 6])
def test_identical_experts_give_single_ffn_for_any_routing(K):
    rng = _rng(22 + K)
    T, H, E, D = 29, 24, 6, 40
    x, wr, _, _, ws1, ws2 = _rand_layer(rng, T, H, E, D, Ds=16)
    w1 = np.repeat(rng.normal(size=(1, D, H)) / math.sqrt(H), E, 0)
    w2 = np.repeat(rng.normal(size=(1, H, D)) / math.sqrt(D), E, 0)
    bias = rng.uniform(-1, 1, size=E)
    out = oracle.moe_layer_forward(x, wr, bias, w1, w2, ws1, ws2, K)
    np.testing.assert_allclose(out["y"], _torch_ffn(x, w1[0], w2[0]) + _torch_ffn(x, ws1, ws2),
                               rtol=1e-11, atol=1e-12)


def test_K1_is_an_identity_scatter_of_the_chosen_expert():
    rng = _rng(23)
    T, H, E, D = 40, 16, 5, 24
    x, wr, w1, w2, _, _ = _rand_layer(rng, T, H, E, D)
    out = oracle.moe_layer_forward(x, wr, None, w1, w2, None, None, 1)
    for t in range(T):
        e = out["idx"][t, 0]
        np.testing.assert_allclose(out["y"][t], _torch_ffn(x[t:t + 1], w1[e], w2[e])[0],
                                   rtol=1e-12, atol=1e-13)


def test_given_logits_decide_the_routing():
    """With caller-given logits the selection follows them, not x W_r^T: a
    one-hot logit row sends every token to its expert (K=1 gives exactly that
    expert's FFN), and with K=2 the weights are the renormalised softmax of
    the two given scores (closed form 1/(1+e^-d))."""
    rng = _rng(26)
    T, H, E, D = 23, 16, 6, 20
    x, wr, w1, w2, _, _ = _rand_layer(rng, T, H, E, D)
    hot = rng.integers(0, E, size=T)
    lg = np.full((T, E), -3.0)
    lg[np.arange(T), hot] = 2.0
    out = oracle.moe_layer_forward(x, wr, None, w1, w2, None, None, 1, logits=lg)
    assert (out["idx"][:, 0] == hot).all()
    assert (out["counts"] == np.bincount(hot, minlength=E)).all()
    for t in range(T):
        np.testing.assert_allclose(out["y"][t], _torch_ffn(x[t:t + 1], w1[hot[t]], w2[hot[t]])[0],
                                   rtol=1e-12, atol=1e-13)
    # K = 2: second-best score 2.0 - d on the next expert (cyclically)
    d = 0.75
    lg2 = lg.copy()
    lg2[np.arange(T), (hot + 1) % E] = 2.0 - d
    out2 = oracle.moe_layer_forward(x, wr, None, w1, w2, None, None, 2, logits=lg2)
    assert (out2["idx"][:, 0] == hot).all() and (out2["idx"][:, 1] == (hot + 1) % E).all()
    np.testing.assert_allclose(out2["w"][:, 0], 1.0 / (1.0 + math.exp(-d)), rtol=1e-7)
    # the router's own logits route differently on this input
    own = oracle.moe_layer_forward(x, wr, None, w1, w2, None, None, 1)
    assert (own["idx"][:, 0] != hot).any()


def test_layer_sum_over_k_matches_explicit_per_token_loop():
    """y[t] = sum_k w[t,k] * FFN_{idx[t,k]}(x[t]) (+ shared), token by token."""
    rng = _rng(24)
    T, H, E, D, K = 17, 20, 7, 28, 3
    x, wr, w1, w2, ws1, ws2 = _rand_layer(rng, T, H, E, D, Ds=12)
    bias = rng.uniform(-0.5, 0.5, size=E)
    out = oracle.moe_layer_forward(x, wr, bias, w1, w2, ws1, ws2, K)
    for t in range(T):
        acc = _torch_ffn(x[t:t + 1], ws1, ws2)[0]
        for k in range(K):
            e = out["idx"][t, k]
            acc = acc + out["w"][t, k] * _torch_ffn(x[t:t + 1], w1[e], w2[e])[0]
        np.testing.assert_allclose(out["y"][t], acc, rtol=1e-12, atol=1e-13)


def test_permutation_equivariance():
    rng = _rng(25)
    T, H, E, D, K = 31, 16, 9, 20, 2
    x, wr, w1, w2, ws1, ws2 = _rand_layer(rng, T, H, E, D, Ds=8)
    p = rng.permutation(T)
    a = oracle.moe_layer_forward(x, wr, None, w1, w2, ws1, ws2, K)["y"]
    b = oracle.moe_layer_forward(x[p], wr, None, w1, w2, ws1, ws2, K)["y"]
    np.testing.assert_allclose(b, a[p], rtol=1e-12, atol=1e-13)


def test_token_subset_equals_rows_of_full_output():
    rng = _rng(26)
    x, wr, w1, w2, ws1, ws2 = _rand_layer(rng, 45, 16, 6, 20, Ds=8)
    full = oracle.moe_layer_forward(x, wr, None, w1, w2, ws1, ws2, 2)
    sub = np.array([0, 3, 4, 20, 44])
    part = oracle.moe_layer_forward(x, wr, None, w1, w2, ws1, ws2, 2, tokens=sub)
    np.testing.assert_allclose(part["y"], full["y"][sub], rtol=0, atol=0)


def test_routed_output_is_linear_in_w2():
    rng = _rng(27)
    x, wr, w1, w2, _, _ = _rand_layer(rng, 12, 16, 4, 20)
    a = oracle.moe_layer_forward(x, wr, None, w1, w2, None, None, 2)["y"]
    b = oracle.moe_layer_forward(x, wr, None, w1, 2.0 * w2, None, None, 2)["y"]
    np.testing.assert_allclose(b, 2.0 * a, rtol=1e-14, atol=0)


# ----------------------------------------------------------------- stats ---
def _golden():
    with open(os.path.join(GOLDEN, "load_stats_cases.json")) as f:
        return json.load(f)


def test_gini_golden_cases():
    for case in _golden()["gini"]:
        want = case["gini"] if "gini" in case else case["gini_num"] / case["gini_den"]
        assert oracle.gini_exact(np.array(case["counts"])) == pytest.approx(want, abs=1e-15)
        assert oracle.gini_page_form(np.array(case["counts"])) == pytest.approx(want, abs=1e-14)


def test_gini_matches_mean_absolute_difference_form():
    rng = _rng(31)
    for n in (2, 3, 8, 128, 256):
        for _ in range(5):
            c = rng.integers(0, 50, size=n) * (rng.random(n) < 0.7)
            if c.sum() == 0:
                continue
            mad = np.abs(c[:, None] - c[None, :]).sum() / (2.0 * n * n * c.mean())
            assert oracle.gini_exact(c) == pytest.approx(mad, abs=1e-13)
            assert oracle.gini_exact(c) == pytest.approx(oracle.gini_page_form(c), abs=1e-14)
    assert oracle.gini_exact(np.full(64, 7)) == 0.0
    for n in (1, 2, 16, 256):
        one_hot = np.zeros(n, dtype=np.int64)
        one_hot[n // 2] = 1000
        assert oracle.gini_exact(one_hot) == pytest.approx((n - 1) / n, abs=1e-15)


def test_max_over_mean_closed_forms():
    """Hottest expert over the mean load T*K/E: 1 for an even load, E when a
    single copy exists, and a hand-worked uneven case."""
    assert oracle.load_stats(np.full(8, 5), 20, 2)["max_over_mean"] == 1.0
    assert oracle.load_stats(np.eye(1, 16, 3, dtype=np.int64)[0], 1, 1)["max_over_mean"] == 16.0
    assert oracle.load_stats(np.array([1, 2, 3, 4]), 5, 2)["max_over_mean"] == 1.6   # 4 / (10/4)
    assert oracle.load_stats(np.zeros(4, np.int64), 0, 2)["max_over_mean"] == 0.0


def test_load_stats_golden_cases():
    for case in _golden()["stats"]:
        T, K = case["T"], case["K"]
        if "counts" in case:
            counts = np.array(case["counts"])
        else:
            counts = np.zeros(case["E"], dtype=np.int64)
            counts[case["hot"]] = 1
        st = oracle.load_stats(counts, T, K)
        for key in ("capacity", "max_load", "min_load", "overflow", "num_stragglers"):
            assert st[key] == case[key], key
        assert st["overflow_rate"] == pytest.approx(case["overflow_rate"], abs=1e-15)
        assert st["skew_ratio"] == pytest.approx(case["max_load"] / (case["min_load"] + 1e-5), rel=1e-15)
        if "straggler_mask" in case:
            assert st["straggler_mask"].tolist() == case["straggler_mask"]


def test_capacity_integer_form_equals_page_float_form():
    for wl in mi.WORKLOADS.values():
        for T in wl.Ts + (0, 1, 3, 1000, 65536):
            assert oracle.capacity(T, wl.K, wl.E) == oracle.capacity_page_float(T, wl.K, wl.E)


def test_stats_on_a_routed_batch_are_consistent():
    rng = _rng(33)
    T, E, K = 256, 64, 8
    idx, _, _ = oracle.select_topk(rng.normal(size=(T, E)), -0.5 * np.log(np.arange(E) + 1.0), K)
    counts = oracle.expert_counts(idx, E)
    st = oracle.load_stats(counts, T, K)
    cap = st["capacity"]
    assert st["overflow"] == sum(max(0, int(c) - cap) for c in counts)
    assert st["num_stragglers"] == int(st["straggler_mask"].sum())
    assert 0.0 <= st["gini"] < 1.0


# ------------------------------------------------ stage-wise formulation ---
def test_stagewise_grouped_ffn_and_combine_equal_layer_definition():
    """Dispatch -> per-expert FFN on each segment -> combine gives the same y
    as the per-token definition, including idle experts and the shared one."""
    rng = _rng(41)
    T, H, E, D, K = 23, 16, 9, 20, 3
    x, wr, w1, w2, ws1, ws2 = _rand_layer(rng, T, H, E, D, Ds=12)
    bias = -0.8 * np.log(np.arange(E) + 1.0)
    out = oracle.moe_layer_forward(x, wr, bias, w1, w2, ws1, ws2, K)
    y_rows, y_sh = oracle.grouped_ffn(x, out["perm"], out["offsets"], K, w1, w2, ws1, ws2)
    for r in range(T * K):                       # row r is copy perm[r] of token perm[r] // K
        e = np.searchsorted(out["offsets"], r, side="right") - 1
        np.testing.assert_allclose(y_rows[r], _torch_ffn(x[out["perm"][r] // K][None], w1[e], w2[e])[0],
                                   rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(oracle.combine(y_rows, out["w"], out["inv"], y_sh), out["y"],
                               rtol=1e-12, atol=1e-13)


def test_combine_worked_example():
    """Two tokens, K = 2, H = 2, by hand: y[t] = sum_k w[t,k] * rows[inv[t*K+k]] + shared[t]."""
    rows = np.array([[1.0, -1.0], [2.0, 0.0], [3.0, 1.0], [4.0, 2.0]])
    inv = np.array([2, 0, 3, 1])                  # copy c of token c // 2 sits in row inv[c]
    w = np.array([[0.25, 0.75], [0.5, 0.5]])
    shared = np.array([[10.0, 20.0], [30.0, 40.0]])
    y = oracle.combine(rows, w, inv)
    np.testing.assert_array_equal(y, [[0.25 * 3 + 0.75 * 1, 0.25 * 1 + 0.75 * -1],
                                      [0.5 * 4 + 0.5 * 2, 0.5 * 2 + 0.5 * 0]])
    np.testing.assert_array_equal(oracle.combine(rows, w, inv, shared), y + shared)


def test_combine_K1_unit_weight_is_inverse_permutation():
    rng = _rng(42)
    TK, H = 19, 5
    rows = rng.normal(size=(TK, H))
    perm = rng.permutation(TK)
    inv = np.empty(TK, dtype=np.int64)
    inv[perm] = np.arange(TK)
    y = oracle.combine(rows, np.ones((TK, 1)), inv)
    np.testing.assert_array_equal(y, rows[inv])


# ------------------------------------------------------------ bias update ---
def test_bias_update_moves_only_overloaded_and_idle_experts():
    counts = np.array([30, 0, 5, 10, 0, 11])           # T=16, K=3, E=6: capacity = 48*5//24 = 10
    b = np.array([0.0, 0.5, -0.25, 1.0, 0.0, -1.0], np.float32)
    nb = oracle.bias_update(b, counts, 16, 3, 0.125)
    assert oracle.capacity(16, 3, 6) == 10
    assert nb.tolist() == [-0.125, 0.625, -0.25, 1.0, 0.125, -1.125]
    assert nb.dtype == np.float32


def test_bias_update_is_a_fixed_point_for_an_even_load():
    counts = np.full(16, 8)
    b = np.linspace(-1, 1, 16).astype(np.float32)
    assert (oracle.bias_update(b, counts, 64, 2, 0.01) == b).all()


def test_repeated_bias_updates_even_out_a_skewed_router():
    """The page's stated purpose: routing with the updated bias spreads the
    load (Gini falls) without retraining the gate."""
    rng = _rng(51)
    T, E, K = 512, 32, 4
    logits = rng.normal(size=(T, E)) - 0.6 * np.log(np.arange(E) + 1.0)
    b = np.zeros(E, np.float32)
    g0 = oracle.gini_exact(oracle.expert_counts(oracle.select_topk(logits, b, K)[0], E))
    for _ in range(60):
        counts = oracle.expert_counts(oracle.select_topk(logits, b, K)[0], E)
        b = oracle.bias_update(b, counts, T, K, 0.02)
    g1 = oracle.gini_exact(oracle.expert_counts(oracle.select_topk(logits, b, K)[0], E))
    assert g1 < 0.6 * g0


# ------------------------------------------------------ Gumbel-noise routing ---
def _gumbel(rng, shape):
    u = rng.uniform(size=shape)
    return (-np.log(-np.log(u))).astype(np.float32)


def test_noisy_routing_without_noise_is_plain_routing():
    rng = np.random.default_rng(5)
    l = rng.normal(size=(40, 12))
    b = rng.uniform(-0.3, 0.3, 12).astype(np.float32)
    i0, w0, s0 = oracle.select_topk(l, b, 3)
    i1, w1, s1 = oracle.select_topk(l, b, 3, noise=np.zeros((40, 12), np.float32))
    assert (i0 == i1).all() and np.array_equal(w0, w1) and np.array_equal(s0, s1)


def _softmax(v):
    z = np.exp(v - v.max())
    return z / z.sum()


def test_gumbel_max_picks_each_expert_with_its_softmax_probability():
    """Gumbel-max: argmax_e (l_e + B_e + g_e) with standard Gumbel g is e with
    probability softmax(l + B)_e (the selection probabilities the page's
    noisy softmax routing gives at K = 1)."""
    rng = np.random.default_rng(11)
    E, N = 5, 200_000
    l = np.array([0.3, -0.4, 1.1, 0.0, -1.5])
    b = np.array([0.1, 0.2, -0.3, 0.0, 0.25], np.float32)
    p = _softmax(l + b.astype(np.float64))
    idx, w, _ = oracle.select_topk(np.tile(l, (N, 1)), b, 1, noise=_gumbel(rng, (N, E)))
    freq = np.bincount(idx[:, 0], minlength=E) / N
    assert np.all(np.abs(freq - p) <= 5 * np.sqrt(p * (1 - p) / N))
    assert np.all(w == 1.0)


def test_gumbel_top2_follows_plackett_luce_order():
    """Gumbel-top-k: the first two slots are experts a then b with
    probability p_a * p_b / (1 - p_a) (sampling without replacement in
    proportion to softmax(l + B))."""
    rng = np.random.default_rng(12)
    E, N = 4, 200_000
    l = np.array([0.5, -0.2, 0.9, -1.0])
    p = _softmax(l)
    idx, _, _ = oracle.select_topk(np.tile(l, (N, 1)), None, 2, noise=_gumbel(rng, (N, E)))
    pair = idx[:, 0] * E + idx[:, 1]
    freq = np.bincount(pair, minlength=E * E) / N
    for a in range(E):
        for c in range(E):
            q = 0.0 if a == c else p[a] * p[c] / (1 - p[a])
            assert abs(freq[a * E + c] - q) <= 5 * math.sqrt(max(q * (1 - q), 1e-12) / N) + 1e-12


def test_noisy_weights_are_the_softmax_of_the_noisy_scores():
    rng = np.random.default_rng(13)
    l = rng.normal(size=(30, 9))
    b = rng.uniform(-0.5, 0.5, 9).astype(np.float32)
    g = _gumbel(rng, (30, 9))
    idx, w, s = oracle.select_topk(l, b, 4, noise=g)
    want = ((l.astype(np.float32) + b).astype(np.float32) + g).astype(np.float32)
    assert np.array_equal(s, want)
    sel = np.take_along_axis(s.astype(np.float64), idx, 1)
    assert np.all(np.diff(sel, axis=1) <= 0)                      # slots by descending noisy score
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-12)
    np.testing.assert_allclose(w[:, 1:] / w[:, :1], np.exp(sel[:, 1:] - sel[:, :1]), rtol=1e-12)
