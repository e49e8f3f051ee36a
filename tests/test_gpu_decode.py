"""The single-launch decode forward (bf16 layers, T <= 2 tokens) against the
fp64 oracle, through moe_layer_forward.

moe_layer_forward runs such batches as one cooperative kernel (router GEMV,
top-K and dispatch in every CTA, weight-streaming expert layers, fused
combine). The oracle is routed from the kernel's fp32 logits, so routing,
dispatch and statistics must be bit-identical on every token; the output
within the bf16 tolerance. Shapes cover the workloads' layers, row lengths
that are not a whole number of 32-vector lane rounds (H = 384), long rows (D = 14336), the
largest copy count (T = 2, K = 16), a single expert, no shared expert, the
Gumbel-noise variant and CUDA-graph replay.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from parity import DeviceLayer, check_layer, routing_buffers, routing_np, to_np

pytestmark = pytest.mark.gpu

_cache = {}


@pytest.fixture(scope="module")
def M():
    from _lib import build_and_import
    return build_and_import()


def layer(wl):
    key = (wl.key, wl.H, wl.E, wl.K, wl.D, wl.Ds)
    if key not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        _cache[key] = DeviceLayer(wl)
    return _cache[key]


def forward(M, L, T, replica=0, noise=None, ws=None):
    wl = L.wl
    x = mi.draw_x(wl, T, replica)
    xd = x.cuda()
    d = L.desc(M, T)
    if ws is None:
        ws = M.alloc_workspace(d)
    r = routing_buffers(wl, T)
    y = torch.full_like(xd, float("nan"))
    n0 = M.moe_kernel_launch_count()
    if noise is None:
        M.moe_layer_forward(d, L.weights(M), xd, y, M.make_routing(**r), ws)
    else:
        M.moe_layer_forward_noisy(d, L.weights(M), xd, noise.cuda(), y, M.make_routing(**r), ws)
    launches = M.moe_kernel_launch_count() - n0
    torch.cuda.synchronize()
    assert M.moe_check_status(ws) == 0
    return x, y, r, ws, launches


SHAPES = [
    ("c3", {}, (1, 2)),
    ("c2", {}, (1,)),
    ("c4", {}, (1, 2)),
    ("c3", dict(H=384, D=640, Ds=1152), (1, 2)),     # rows not a multiple of 32 vectors
    ("c3", dict(H=256, E=512, K=16, D=256, Ds=0), (2,)),   # 32 copies, no shared expert
    ("c3", dict(H=128, E=1, K=1, D=128, Ds=128), (1, 2)),  # one expert
]


@pytest.mark.parametrize("key,shape,Ts", SHAPES)
def test_decode_forward_matches_oracle(M, key, shape, Ts):
    wl = mi.with_shape(mi.WORKLOADS[key], **shape)
    L = layer(wl)
    for T in Ts:
        x, y, r, ws, launches = forward(M, L, T)
        assert launches == 1, f"T={T}: {launches} launches, expected one"
        d = L.desc(M, T)
        mask = torch.empty(wl.E, dtype=torch.uint8, device="cuda")
        st = M.moe_expert_stats(d, r["counts"], mask, ws)
        check_layer(wl, x, L, routing_np(r), to_np(y), stats=st, mask=to_np(mask))


@pytest.mark.parametrize("key,T", [("c3", 3), ("c4", 4), ("c2", 2)])
def test_larger_batches_take_the_multi_launch_path(M, key, T):
    # beyond two tokens (c3, c4), or where the staged activations exceed the
    # shared memory beside the weight ring (c2 T=2), the multi-launch path runs them
    wl = mi.WORKLOADS[key]
    L = layer(wl)
    x, y, r, ws, launches = forward(M, L, T)
    assert launches > 1
    check_layer(wl, x, L, routing_np(r), to_np(y))


def test_decode_forward_is_deterministic_and_reuses_its_workspace(M):
    L = layer(mi.WORKLOADS["c3"])
    x, y0, r0, ws, _ = forward(M, L, 2)
    for rep in range(3):          # same workspace: the barrier counters start from zero again
        _, y1, r1, _, _ = forward(M, L, 2, ws=ws)
        assert torch.equal(y0, y1)
        for k in r0:
            assert torch.equal(r0[k], r1[k]), k
    # status word and the header's arrival counters (the grid barrier) are back at zero
    hdr = ws[:256].view(torch.int32)
    assert hdr[0] == 0 and (hdr[5:13] == 0).all(), "control words not left at zero"


def test_decode_noisy_forward_matches_oracle(M):
    wl = mi.with_shape(mi.WORKLOADS["c4"], H=512, D=256, Ds=512)
    L = layer(wl)
    T = 2
    g = mi.draw_gumbel(T, wl.E, seed=wl.seed + 77)
    x, y, r, _, launches = forward(M, L, T, noise=g)
    assert launches == 1
    check_layer(wl, x, L, routing_np(r), to_np(y), noise=g.numpy())


def test_decode_graph_replay_equals_eager(M):
    wl = mi.with_shape(mi.WORKLOADS["c3"], H=512, D=256, Ds=512)
    L = layer(wl)
    T = 1
    d = L.desc(M, T)
    W = L.weights(M)
    xs = mi.draw_x(wl, T, 0).cuda()
    ys = torch.empty_like(xs)
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
        g.replay()
        ye = torch.empty_like(xs)
        re = routing_buffers(wl, T)
        M.moe_layer_forward(d, W, xs, ye, M.make_routing(**re), ws_e)
        torch.cuda.synchronize()
        assert torch.equal(ys, ye)
        for k in rs:
            assert torch.equal(rs[k], re[k]), k
        check_layer(wl, x, L, routing_np(rs), to_np(ys))
    assert M.moe_check_status(ws) == 0
    del g
