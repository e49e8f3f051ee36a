"""moe_layer_forward captured in a CUDA graph and replayed: every replay must
equal the eager call on the same input bit for bit (the path has no atomics
in its arithmetic and no host decisions that depend on data), and match the
oracle. Covers the one-CTA dispatch, split-K router/GEMM2, the CTA-pair GEMMs
and the fp32 CUDA-core path, plus a bias update captured with the forward."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from parity import DeviceLayer, compare_routing, rel_max_err, to_np, y_tol

pytestmark = pytest.mark.gpu

CASES = [
    ("c1", {}, 64),                                        # fp32, CUDA cores
    ("c3", dict(H=512, D=256, Ds=512), 1),                 # decode: split-K router + GEMM2
    ("c3", dict(H=512, D=256, Ds=512), 40),
    ("c2", dict(H=512, D=1024), 300),                      # 64+ rows per expert: CTA pairs
    ("c4", dict(H=256, D=128, Ds=256), 3000),              # multi-chunk dispatch
]


@pytest.fixture(scope="module")
def M():
    from _lib import build_and_import
    return build_and_import()


def _routing(wl, T):
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


@pytest.mark.parametrize("key,shape,T", CASES)
def test_graph_replay_equals_eager(M, key, shape, T):
    wl = mi.with_shape(mi.WORKLOADS[key], **shape)
    L = DeviceLayer(wl)
    d = L.desc(M, T)
    W = L.weights(M)
    xs = mi.draw_x(wl, T, 0).cuda()
    ys = torch.full_like(xs, float("nan"))
    rs = _routing(wl, T)
    ws = M.alloc_workspace(d)
    R = M.make_routing(**rs)
    M.moe_layer_forward(d, W, xs, ys, R, ws)             # first call outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        M.moe_layer_forward(d, W, xs, ys, R, ws)
    ws_e = M.alloc_workspace(d)
    for replica in range(3):
        x = mi.draw_x(wl, T, replica)
        xs.copy_(x)
        ys.fill_(float("nan"))
        g.replay()
        ye = torch.full_like(xs, float("nan"))
        re = _routing(wl, T)
        M.moe_layer_forward(d, W, xs, ye, M.make_routing(**re), ws_e)
        torch.cuda.synchronize()
        assert torch.equal(ys, ye), f"replay {replica} differs from the eager call"
        for k in rs:
            assert torch.equal(rs[k], re[k]), k
        if replica == 0:
            ref = oracle.moe_layer_forward(mi.to_f64(x), L.wr64, L.bias, L.w1_64, L.w2_64,
                                           L.ws1_64, L.ws2_64, wl.K)
            uniq, _, _ = compare_routing(wl, to_np(rs["logits"]), to_np(rs["topk_idx"]),
                                         to_np(rs["topk_w"]), ref["logits"], L.bias)
            err = rel_max_err(to_np(ys)[uniq], ref["y"][uniq])
            assert err <= y_tol(wl), f"max |y - y_ref| = {err:.3e} x RMS"
    assert M.moe_check_status(ws) == 0 and M.moe_check_status(ws_e) == 0
    del g


def test_graph_with_bias_update(M):
    """Forward + bias update captured together: the bias evolves across
    replays exactly as in the eager sequence and as the oracle computes."""
    wl = mi.with_shape(mi.WORKLOADS["c3"], H=256, D=128, Ds=256)
    T, gamma, steps = 64, 0.01, 6
    L = DeviceLayer(wl)
    d = L.desc(M, T)
    xs = mi.draw_x(wl, T, 0).cuda()
    ys = torch.empty_like(xs)
    rs = _routing(wl, T)
    ws = M.alloc_workspace(d)
    R = M.make_routing(**rs)
    bias0 = L.dev["bias"].clone()

    def step(b, x, y, r, R_, w):
        W = M.make_weights(L.dev["w_router"], L.dev["w1"], L.dev["w2"], L.dev["ws1"],
                           L.dev["ws2"], b)
        M.moe_layer_forward(d, W, x, y, R_, w)
        M.moe_bias_update(d, r["counts"], b, gamma)

    b_g = bias0.clone()
    step(b_g, xs, ys, rs, R, ws)                         # first call outside capture
    torch.cuda.synchronize()
    b_g.copy_(bias0)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(b_g, xs, ys, rs, R, ws)
    torch.cuda.synchronize()
    b_g.copy_(bias0)                                     # capture does not run the kernels
    b_e = bias0.clone()
    re = _routing(wl, T)
    ws_e = M.alloc_workspace(d)
    ye = torch.empty_like(xs)
    b_ref = L.bias.copy()
    for s in range(steps):
        x = mi.draw_x(wl, T, s)
        xs.copy_(x)
        g.replay()
        step(b_e, xs, ye, re, M.make_routing(**re), ws_e)
        torch.cuda.synchronize()
        assert torch.equal(b_g, b_e) and torch.equal(ys, ye)
        uniq, _, _ = compare_routing(wl, to_np(rs["logits"]), to_np(rs["topk_idx"]),
                                     to_np(rs["topk_w"]),
                                     oracle.router_logits(mi.to_f64(x), L.wr64), b_ref)
        if uniq.all():
            ref_idx, _, _ = oracle.select_topk(oracle.router_logits(mi.to_f64(x), L.wr64), b_ref,
                                               wl.K)
            b_ref = oracle.bias_update(b_ref, oracle.expert_counts(ref_idx, wl.E), T, wl.K, gamma)
            assert (to_np(b_g).view(np.int32) == b_ref.view(np.int32)).all()
        else:
            pytest.skip("near-tied routing decision; the bias trajectories may part")
    del g
