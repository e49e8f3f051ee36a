"""Helpers for comparing the CUDA path with the fp64 oracle.

Routing rule. The kernels compute gate logits in fp32 with their own
summation order, so the fp32 scores s = l + B can differ from the oracle's in
the last bits; the decision is taken in the same precision on both sides
(fp32). A token's selection is *unique* when every adjacent gap among its
K+1 best oracle scores exceeds twice the worst score discrepancy `tol`
(measured logit error plus fp32 rounding); then the chosen experts and slot
order must match exactly. For the other tokens several answers are correct,
and the GPU's choice is checked for validity against the oracle's scores.
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
W_TOL = 1e-6          # max |w - w_ref| of the renormalised weights


def y_tol(wl) -> float:
    return F32_Y_TOL if wl.dtype == "f32" else BF16_Y_TOL


def logit_tol(wl) -> float:
    return F32_LOGIT_TOL if wl.dtype == "f32" else BF16_LOGIT_TOL


def rel_max_err(got: np.ndarray, ref: np.ndarray) -> float:
    rms = float(np.sqrt(np.mean(np.square(ref)))) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(got - ref))) / max(rms, 1e-30)


def scores64(logits64: np.ndarray, bias, noise=None) -> np.ndarray:
    b = np.zeros(logits64.shape[1]) if bias is None else np.asarray(bias, np.float64)
    s = logits64 + b[None, :]
    return s if noise is None else s + np.asarray(noise, np.float64)


def unique_selection_mask(s64: np.ndarray, K: int, tol: float) -> np.ndarray:
    """True where the top-K set and slot order are unique beyond +-tol."""
    E = s64.shape[1]
    srt = -np.sort(-s64, axis=1)[:, :min(K + 1, E)]
    if srt.shape[1] < 2:
        return np.ones(s64.shape[0], dtype=bool)
    gaps = srt[:, :-1] - srt[:, 1:]
    return gaps.min(axis=1) > 2.0 * tol


def check_selection_valid(idx: np.ndarray, s64: np.ndarray, tol: float):
    """The chosen experts are distinct, beat every other expert up to 2*tol,
    and the slots are in descending score order up to 2*tol."""
    T, K = idx.shape
    E = s64.shape[1]
    for t in range(T):
        row = idx[t]
        assert len(set(row.tolist())) == K and row.min() >= 0 and row.max() < E
        chosen = s64[t, row]
        others = np.delete(s64[t], row)
        if others.size:
            assert chosen.min() >= others.max() - 2 * tol
        assert (np.diff(chosen) <= 2 * tol).all()


def compare_routing(wl, gpu_logits, gpu_idx, gpu_w, ref_logits64, bias, noise=None):
    """Returns (unique mask, oracle routing) after checking logits, selection
    and weights as described in the module doc."""
    K = wl.K
    rms = float(np.sqrt(np.mean(ref_logits64 ** 2))) if ref_logits64.size else 1.0
    lerr = float(np.max(np.abs(gpu_logits.astype(np.float64) - ref_logits64))) if ref_logits64.size else 0.0
    assert lerr <= logit_tol(wl) * rms, f"logit error {lerr / rms:.3e} x RMS"
    s64 = scores64(ref_logits64, bias, noise)
    tol = lerr + 2.0 ** -22 * (float(np.abs(s64).max()) if s64.size else 0.0)
    uniq = unique_selection_mask(s64, K, tol)
    ref_idx, ref_w, _ = oracle.select_topk(ref_logits64, bias, K, noise)
    assert (gpu_idx[uniq] == ref_idx[uniq]).all(), "selection differs on a token with a unique answer"
    # w_k = softmax of the chosen scores: dw_k/ds_j = w_k (delta_kj - w_j), so a
    # score error e moves each weight by at most 2 e (plus fp32 rounding).
    w_tol = W_TOL + 2.0 * tol
    assert np.max(np.abs(gpu_w[uniq] - ref_w[uniq]), initial=0.0) <= w_tol
    if (~uniq).any():
        check_selection_valid(gpu_idx[~uniq], s64[~uniq], tol)
    np.testing.assert_allclose(gpu_w.sum(axis=1), 1.0, atol=1e-6)
    return uniq, ref_idx, ref_w


def check_dispatch_valid(idx, counts, offsets, perm, inv, E):
    """Invariants of a correct dispatch of idx (used where the oracle's own
    routing differs on a near-tie token)."""
    T, K = idx.shape
    flat = idx.reshape(-1)
    assert counts.sum() == T * K and (np.diff(offsets) == counts).all() and offsets[0] == 0
    assert (np.sort(perm) == np.arange(T * K)).all() and (inv[perm] == np.arange(T * K)).all()
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert (flat[seg] == e).all() and (np.diff(seg) > 0).all()


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


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy()
