"""The synthetic input recipe against the routing structure it is meant to produce.

The pages measure on real chat traffic through trained weights: a Zipf-like
long tail of expert popularity ("Kimi K3 专家路由不均衡诊断", section 一) and
hot/cold expert hit ratios of 14x-89x ("Kimi K3 专家路由不均衡诊断",
section 二). The seeded stand-ins in moe_inputs draw x ~ N(0, 1),
W_r ~ N(0, 1/H) and add the offset -(1/3) s ln(e + 1) to the bias input.
These tests route the drawn tensors with the oracle and check the structure
that every benchmark point depends on: how many experts a decode batch
touches (which sets its HBM bytes) and how skewed the prefill load is (which
sets the largest expert's tile count). The expected values are those of a
separate numpy simulation of the same recipe; a recipe error (a wrong offset
scale or sign, a wrong router weight scale) moves them well outside the
windows below.
"""
import numpy as np
import pytest

import moe_inputs as mi
import oracle


def _route(wl, T):
    x = mi.to_f64(mi.draw_x(wl, T))
    w_r = mi.to_f64(mi.draw_router(wl))
    b = mi.draw_bias(wl).double().numpy()
    logits = oracle.router_logits(x, w_r).astype(np.float32)
    idx, _, _ = oracle.select_topk(logits, b, wl.K)
    return idx


def _zipf_part(wl):
    e = np.arange(wl.E, dtype=np.float64)
    return -mi.ZIPF_BETA * wl.zipf_s * np.log(e + 1.0)


@pytest.mark.parametrize("key", ["c3", "c5"])
def test_bias_input_is_the_zipf_offset(key):
    wl = mi.WORKLOADS[key]
    b = mi.draw_bias(wl).double().numpy()
    assert b[0] == 0.0                       # expert 0 is the hottest
    assert (np.diff(b) < 0).all()            # strictly decreasing with the index
    # -(1/3) s ln(e + 1), rounded once to fp32
    np.testing.assert_allclose(b[1:] / np.log(np.arange(2, wl.E + 1)), -wl.zipf_s / 3.0,
                               rtol=2 ** -22)


def test_heavy_skew_bias_adds_a_uniform_draw():
    wl = mi.WORKLOADS["c4"]
    b = mi.draw_bias(wl).double().numpy()
    u = b - _zipf_part(wl)
    assert np.abs(u).max() <= wl.bias_uniform + 1e-6
    assert np.abs(u).max() > 0.4             # the draw is there, spread over (-0.5, 0.5)
    assert abs(u.mean()) < 0.1               # 256 draws: mean within ~5 standard errors of 0


# (workload, T, touched experts of the simulation)
TOUCHED = [("c3", 1, 8), ("c3", 16, 73), ("c3", 32, 100), ("c3", 64, 113), ("c3", 128, 125),
           ("c4", 16, 67), ("c4", 64, 156), ("c4", 128, 182), ("c4", 256, 226)]


@pytest.mark.parametrize("key,T,expect", TOUCHED)
def test_decode_batches_touch_the_simulated_number_of_experts(key, T, expect):
    wl = mi.WORKLOADS[key]
    touched = len(np.unique(_route(wl, T)))
    assert touched <= min(wl.E, T * wl.K)
    if T == 1:
        assert touched == wl.K               # one token: K distinct experts
    else:
        assert abs(touched - expect) <= 0.2 * expect, (key, T, touched, expect)


def test_prefill_load_skew_matches_the_simulation():
    """16384 tokens of the 128-expert layer (s = 1.1): the simulation gives a
    hot/cold ratio of ~18x, a Gini coefficient of ~0.39 and ~6.8k rows on
    the hottest expert (against a mean of 1024)."""
    wl = mi.WORKLOADS["c5"]
    T = 16384
    counts = np.bincount(_route(wl, T).ravel(), minlength=wl.E)
    assert counts.sum() == T * wl.K
    assert counts.argmax() == 0
    assert counts.min() > 0
    assert 12 <= counts.max() / counts.min() <= 30
    assert 0.35 <= oracle.gini_exact(counts) <= 0.43
    assert 6000 <= counts.max() <= 7800


def test_heavier_zipf_exponent_and_bias_give_a_more_skewed_load():
    """The 256-expert layer (s = 1.3 plus B ~ U(-0.5, 0.5)) is more skewed
    than the 128-expert one (s = 1.1), as the pages' heavier-load rows are."""
    T = 4096
    g = {}
    for key in ("c4", "c5"):
        wl = mi.WORKLOADS[key]
        g[key] = oracle.gini_exact(np.bincount(_route(wl, T).ravel(), minlength=wl.E))
    assert g["c4"] > g["c5"] + 0.1, g

