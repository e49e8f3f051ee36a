"""Helpers for comparing the CUDA path with the fp64 oracle.

Parity rule. The kernels compute the gate logits in fp32 in their own
summation order, the oracle in fp64; the two sets of logits are compared
with each other within a tolerance (the logit check). The routing is then
checked by re-routing the oracle from the GPU's own fp32 logits, so that both
sides take the top-K decision on identical numbers, in the same precision
(fp32 scores s = l + B). Given the same logits the routing is exact: the
indices, counts, offsets, permutation, inverse permutation and every load
statistic must be bit-identical on every token, and the renormalised weights
within W_TOL. The oracle's expert FFNs and combine then run on that same
routing, and the layer output is compared within the output tolerance on
every token the oracle computes (all of them, or a seeded sample at the
largest token counts).
"""
from __future__ import annotations

import numpy as np
import torch

import moe_inputs as mi
import oracle

BF16_Y_TOL = 2e-2     # max |y - y_ref| / RMS(y_ref) for bf16 layers
F32_Y_TOL = 1e-5      # ... for fp32 layers
BF16_LOGIT_TOL = 1e-4  # max |l - l_ref| / RMS(l_ref) (fp32 accumulation of exact bf16 products)
F32_LOGIT_TOL = 1e-5
W_TOL = 1e-6          # max |w - w_ref| of the renormalised weights from the same logits


def y_tol(wl) -> float:
    return F32_Y_TOL if wl.dtype == "f32" else BF16_Y_TOL


def logit_tol(wl) -> float:
    return F32_LOGIT_TOL if wl.dtype == "f32" else BF16_LOGIT_TOL


def rel_max_err(got: np.ndarray, ref: np.ndarray) -> float:
    rms = float(np.sqrt(np.mean(np.square(ref)))) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(got - ref))) / max(rms, 1e-30)


def check_logits(wl, gpu_logits: np.ndarray, ref_logits64: np.ndarray) -> float:
    """GPU fp32 logits against the oracle's fp64 logits (x W_r^T)."""
    if ref_logits64.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref_logits64 ** 2)))
    err = float(np.max(np.abs(gpu_logits.astype(np.float64) - ref_logits64))) / max(rms, 1e-30)
    assert err <= logit_tol(wl), f"logit error {err:.3e} x RMS"
    return err


def check_routing(g: dict, ref: dict, E: int):
    """Routing from the same logits: bit-exact on every token."""
    T, K = ref["idx"].shape
    assert (g["topk_idx"] == ref["idx"]).all(), "top-K indices differ from the oracle's"
    assert np.max(np.abs(g["topk_w"] - ref["w"]), initial=0.0) <= W_TOL, "top-K weights"
    np.testing.assert_allclose(g["topk_w"].sum(axis=1), 1.0, atol=1e-6)
    for k in ("counts", "offsets", "perm", "inv"):
        if k in g:
            assert (g[k] == ref[k]).all(), f"{k} differs from the oracle's"


def check_layer(wl, x_host: torch.Tensor, L, g: dict, y: np.ndarray, bias=None, tokens=None,
                noise=None, stats=None, mask=None) -> dict:
    """The whole parity rule for one forward: `g` holds the GPU's routing
    outputs as numpy arrays (logits, topk_idx, topk_w and, when recorded,
    counts, offsets, perm, inv), `y` its output [T, H]. Returns the oracle's
    result with the measured errors."""
    T, K, E = x_host.shape[0], wl.K, wl.E
    x64 = mi.to_f64(x_host)
    b = L.bias if bias is None else bias
    lerr = check_logits(wl, g["logits"], oracle.router_logits(x64, L.wr64))
    ref = oracle.moe_layer_forward(x64, L.wr64, b, L.w1_64, L.w2_64, L.ws1_64, L.ws2_64, K,
                                   tokens=tokens, noise=noise, logits=g["logits"])
    check_routing(g, ref, E)
    want = oracle.load_stats(ref["counts"], T, K)
    if stats is not None:
        stats_equal(stats, want)
    if mask is not None:
        assert (mask == want["straggler_mask"]).all(), "straggler mask"
    assert not np.isnan(y).any(), "an output element was not written"
    err = rel_max_err(y[ref["tokens"]], ref["y"])
    assert err <= y_tol(wl), f"max |y - y_ref| = {err:.3e} x RMS"
    ref["y_err"], ref["logit_err"] = err, lerr
    return ref


def stats_equal(got: dict, want: dict):
    for k in ("num_copies", "capacity", "max_load", "min_load", "overflow", "num_stragglers"):
        assert int(got[k]) == int(want[k]), k
    for k in ("skew_ratio", "gini", "overflow_rate", "max_over_mean"):
        assert got[k] == want[k], (k, got[k], want[k])     # bit-exact: same exact formula


class DeviceLayer:
    """One workload's weights on the device plus host copies for the oracle."""

    def __init__(self, wl, device="cuda"):
        self.wl = wl
        self.host = mi.draw_layer(wl)
        h = self.host
        self.dev = {k: (v.to(device) if v is not None else None) for k, v in h.items()}
        self.w1_64 = mi.LazyF64(h["w1"])
        self.w2_64 = mi.LazyF64(h["w2"])
        self.wr64 = mi.to_f64(h["w_router"])
        self.ws1_64 = mi.to_f64(h["ws1"])
        self.ws2_64 = mi.to_f64(h["ws2"])
        self.bias = h["bias"].numpy()

    def desc(self, M, T):
        wl = self.wl
        return M.make_desc(T, wl.H, wl.E, wl.K, wl.D, wl.Ds,
                           M.MOE_BF16 if wl.dtype == "bf16" else M.MOE_F32)

    def weights(self, M):
        d = self.dev
        return M.make_weights(d["w_router"], d["w1"], d["w2"], d["ws1"], d["ws2"], d["bias"])


def routing_buffers(wl, T: int) -> dict:
    """Device tensors for every optional routing output of moe_layer_forward."""
    E, K = wl.E, wl.K
    return {
        "topk_idx": torch.empty((T, K), dtype=torch.int32, device="cuda"),
        "topk_w": torch.empty((T, K), dtype=torch.float32, device="cuda"),
        "counts": torch.empty(E, dtype=torch.int32, device="cuda"),
        "offsets": torch.empty(E + 1, dtype=torch.int32, device="cuda"),
        "perm": torch.empty(T * K, dtype=torch.int32, device="cuda"),
        "inv": torch.empty(T * K, dtype=torch.int32, device="cuda"),
        "logits": torch.empty((T, E), dtype=torch.float32, device="cuda"),
    }


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy()


def routing_np(r: dict) -> dict:
    return {k: to_np(v) for k, v in r.items()}
