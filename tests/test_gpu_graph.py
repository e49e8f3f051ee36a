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
from parity import DeviceLayer, check_layer, routing_buffers, routing_np, to_np

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


@pytest.mark.parametrize("key,shape,T", CASES)
def test_graph_replay_equals_eager(M, key, shape, T):
    wl = mi.with_shape(mi.WORKLOADS[key], **shape)
    L = DeviceLayer(wl)
    d = L.desc(M, T)
    W = L.weights(M)
    xs = mi.draw_x(wl, T, 0).cuda()
    ys = torch.full_like(xs, float("nan"))
    rs = routing_buffers(wl, T)
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
        re = routing_buffers(wl, T)
        M.moe_layer_forward(d, W, xs, ye, M.make_routing(**re), ws_e)
        torch.cuda.synchronize()
        assert torch.equal(ys, ye), f"replay {replica} differs from the eager call"
        for k in rs:
            assert torch.equal(rs[k], re[k]), k
        if replica == 0:
            check_layer(wl, x, L, routing_np(rs), to_np(ys))
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
    rs = routing_buffers(wl, T)
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
    re = routing_buffers(wl, T)
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
        # the oracle, routed from the GPU's logits with the bias it held
        # before this step, gives the same counts and so the same new bias
        ref = check_layer(wl, x, L, routing_np(rs), to_np(ys), bias=b_ref)
        b_ref = oracle.bias_update(b_ref, ref["counts"], T, wl.K, gamma)
        assert (to_np(b_g).view(np.int32) == b_ref.view(np.int32)).all()
    del g
