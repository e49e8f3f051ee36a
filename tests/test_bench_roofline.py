"""The benchmark's algorithmic work and roofline bound (CPU only), against
figures worked out by hand from the layer's definition.

FLOPs of one forward: router 2*T*H*E, routed experts 2 GEMMs x 2*H*D per
copy (the Kimi K3 page's Time_comp numerator), shared expert 2 GEMMs x
2*H*Ds per token. HBM bytes: the router matrix, every touched expert's two
matrices, the shared expert's two, x in and y out.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

PEAKS = {"hbm_gbs": 6431.7, "bf16_tflops": 1656.9}


@pytest.mark.parametrize("key,T,touched,flops,nbytes", [
    # Mixtral-shaped layer, one token touching 2 experts: 2*117.4 MB of weights
    ("c2", 1, 2, 2 * 4096 * 8 + 4 * 2 * 4096 * 14336,
     8 * 4096 * 2 + 2 * (2 * 4096 * 14336 * 2) + 2 * 4096 * 2),
    # the headline point: 1.924 TFLOP, all 8 experts' 1.88 GB of weights
    ("c2", 4096, 8, 2 * 4096 * 4096 * 8 + 4 * 4096 * 2 * 4096 * 14336,
     8 * 4096 * 2 + 8 * (2 * 4096 * 14336 * 2) + 2 * 4096 * 4096 * 2),
    # fine-grained decode: 8 of 128 experts plus the 4096-wide shared expert
    ("c3", 1, 8, 2 * 4096 * 128 + 4 * 8 * 4096 * 1024 + 4 * 4096 * 4096,
     128 * 4096 * 2 + 8 * (2 * 4096 * 1024 * 2) + 2 * 4096 * 4096 * 2 + 2 * 4096 * 2),
    # prefill: 3.32 TFLOP (routed 2.20 + shared 1.10 + router 0.017)
    ("c5", 16384, 128, 2 * 16384 * 4096 * 128 + 4 * 16384 * 8 * 4096 * 1024
     + 4 * 16384 * 4096 * 4096,
     128 * 4096 * 2 + 128 * (2 * 4096 * 1024 * 2) + 2 * 4096 * 4096 * 2 + 2 * 16384 * 4096 * 2),
    # the fp32 layer: 4-byte elements
    ("c1", 64, 16, 2 * 64 * 256 * 16 + 4 * 64 * 2 * 256 * 512,
     16 * 256 * 4 + 16 * (2 * 256 * 512 * 4) + 2 * 64 * 256 * 4),
])
def test_algorithmic_work_matches_hand_count(key, T, touched, flops, nbytes):
    import bench
    a = bench.algorithmic(bench.mi.WORKLOADS[key], T, touched)
    assert a["flops"] == flops
    assert a["bytes"] == nbytes


def test_headline_and_prefill_figures():
    import bench
    c2 = bench.algorithmic(bench.mi.WORKLOADS["c2"], 4096, 8)
    assert abs(c2["flops"] / 1e12 - 1.924) < 1e-3
    c5 = bench.algorithmic(bench.mi.WORKLOADS["c5"], 16384, 128)
    assert abs(c5["flops"] / 1e12 - 3.316) < 1e-3


def test_roofline_bound_picks_the_slower_resource():
    import bench
    wl = bench.mi.WORKLOADS
    # decode: HBM-bound, t = bytes / 6431.7 GB/s (c3 T=1: 0.20 GB -> ~31 us)
    a = bench.algorithmic(wl["c3"], 1, 8)
    bound, t = bench.roofline_bound(a["flops"], a["bytes"], PEAKS)
    assert bound == "hbm" and abs(t - a["bytes"] / 6431.7e9) < 1e-12 and 30e-6 < t < 33e-6
    # prefill: tensor-bound, t = flops / 1656.9 TFLOP/s (c5: ~2.0 ms)
    a = bench.algorithmic(wl["c5"], 16384, 128)
    bound, t = bench.roofline_bound(a["flops"], a["bytes"], PEAKS)
    assert bound == "tensor" and abs(t - a["flops"] / 1656.9e12) < 1e-12 and 1.9e-3 < t < 2.1e-3
    # the Mixtral-shaped layer crosses over between T = 512 and T = 4096
    assert bench.roofline_bound(**_fb(bench, wl["c2"], 512, 8))[0] == "hbm"
    assert bench.roofline_bound(**_fb(bench, wl["c2"], 4096, 8))[0] == "tensor"


def _fb(bench, w, T, touched):
    a = bench.algorithmic(w, T, touched)
    return {"flops": a["flops"], "nbytes": a["bytes"], "peaks": PEAKS}


class _FakeRunner:
    def __init__(self, gemm_ms):
        self.gemm_ms = gemm_ms

    def timed_gemms(self, steps):
        return self.gemm_ms


def test_dominant_kernel_roofline_from_the_gemm_loop():
    """achieved = the GEMMs' algorithmic FLOPs / their own loop time; the pair
    must fit in the step that contains it, and a single-launch step is its
    own dominant kernel."""
    import bench
    wl = bench.mi.WORKLOADS["c2"]
    a = bench.algorithmic(wl, 4096, 8)
    peaks = dict(PEAKS, bf16_tflops_sustained=1425.2)
    r = bench.gemm_roofline(_FakeRunner(1.60), wl, 4096, a, peaks, 20, ms_step=1.75)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(a["gemm_flops"] / 1.60e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1656.9)
    assert r["within_step"] and r["share_of_step"] == pytest.approx(1.60 / 1.75)
    assert not bench.gemm_roofline(_FakeRunner(1.80), wl, 4096, a, peaks, 20, 1.75)["within_step"]
    d = bench.algorithmic(bench.mi.WORKLOADS["c3"], 1, 8)
    r = bench.gemm_roofline(_FakeRunner(None), bench.mi.WORKLOADS["c3"], 1, d, peaks, 20, 0.040)
    assert r["bound"] == "hbm" and r["achieved"] == pytest.approx(d["bytes"] / 40e-6 / 1e9)
    assert r["share_of_step"] == 1.0 and r["ms_per_launch_pair"] is None


def test_reference_arm_and_cpu_baseline_share_one_sampling_rule():
    import bench
    wl = bench.mi.WORKLOADS
    assert bench.oracle_sample_size(wl["c2"], 8) == 8
    assert bench.oracle_sample_size(wl["c2"], 4096) == 64
    assert bench.oracle_sample_size(wl["c5"], 16384) == 128
    # both arms describe the same per-step program
    t = bench.oracle_sample_text(wl["c2"], 4096, 20)
    assert "all 4096 tokens" in t and "64 seeded sample tokens" in t
