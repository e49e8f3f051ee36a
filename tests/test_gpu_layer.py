"""Whole-layer parity (moe_layer_forward through the C ABI) on every workload,
against the fp64 oracle on the same seeded inputs.

The oracle is routed from the GPU's own fp32 logits (which are checked
against the oracle's fp64 logits separately), so routing, dispatch and load
statistics must be bit-identical on every token, with no exceptions for
near-ties. Small token counts compare the output on every token; the large
ones (T = 512 and 4096 of the Mixtral-shaped layer, T = 16384 of the prefill
layer) on a seeded sample of tokens the oracle computes one by one, while
routing, dispatch and statistics still cover all tokens. Launch
configuration and workspace are the ones the benchmark uses.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from parity import DeviceLayer, check_layer, routing_buffers, routing_np, to_np

pytestmark = pytest.mark.gpu

FULL_POINTS = [("c1", 64), ("c2", 1), ("c2", 8), ("c2", 64), ("c3", 1), ("c3", 16), ("c3", 32),
               ("c3", 64), ("c3", 128), ("c4", 16), ("c4", 64), ("c4", 128), ("c4", 256)]
SAMPLED_POINTS = [("c2", 512, 64), ("c2", 4096, 64), ("c5", 16384, 128)]

_cache = {}


@pytest.fixture(scope="module")
def M():
    from _lib import build_and_import
    return build_and_import()


def layer(key):
    if key not in _cache:
        _cache.clear()                     # keep one workload's weights resident at a time
        torch.cuda.empty_cache()
        _cache[key] = DeviceLayer(mi.WORKLOADS[key])
    return _cache[key]


def run_and_check(M, L, T, sample=None, replica=0):
    wl = L.wl
    x = mi.draw_x(wl, T, replica)
    xd = x.cuda()
    d = L.desc(M, T)
    ws = M.alloc_workspace(d)
    r = routing_buffers(wl, T)
    y = torch.full_like(xd, float("nan"))
    M.moe_layer_forward(d, L.weights(M), xd, y, M.make_routing(**r), ws)
    torch.cuda.synchronize()
    assert M.moe_check_status(ws) == 0
    mask = torch.empty(wl.E, dtype=torch.uint8, device="cuda")
    st = M.moe_expert_stats(d, r["counts"], mask, ws)
    tokens = None if sample is None else mi.sample_tokens(T, sample, wl.seed + T).numpy()
    ref = check_layer(wl, x, L, routing_np(r), to_np(y), tokens=tokens, stats=st, mask=to_np(mask))
    return ref["y_err"]


@pytest.mark.parametrize("key,T", FULL_POINTS)
def test_layer_all_tokens(M, key, T):
    run_and_check(M, layer(key), T)


@pytest.mark.parametrize("key,T,n", SAMPLED_POINTS)
def test_layer_sampled_tokens(M, key, T, n):
    run_and_check(M, layer(key), T, sample=n)


def test_layer_is_deterministic_and_writes_every_output(M):
    L = layer("c1")
    T = 64
    d = L.desc(M, T)
    ws = M.alloc_workspace(d)
    x = mi.draw_x(L.wl, T).cuda()
    ys = []
    for fill in (float("nan"), 12345.0):
        y = torch.full_like(x, fill)
        M.moe_layer_forward(d, L.weights(M), x, y, None, ws)
        ys.append(y)
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1])


def test_layer_ignores_stale_workspace_contents(M):
    L = layer("c1")
    T = 64
    d = L.desc(M, T)
    ws = M.alloc_workspace(d)
    x = mi.draw_x(L.wl, T).cuda()
    y0 = torch.empty_like(x)
    M.moe_layer_forward(d, L.weights(M), x, y0, None, ws)
    ws[256:].fill_(0xA5)                      # poison everything past the control header
    y1 = torch.empty_like(x)
    M.moe_layer_forward(d, L.weights(M), x, y1, None, ws)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)


@pytest.mark.parametrize("dtype,E,K,Ds", [("f32", 1, 1, 0), ("bf16", 1, 1, 128), ("f32", 6, 6, 0),
                                          ("bf16", 16, 16, 0), ("bf16", 64, 4, 256)])
def test_layer_edge_shapes(M, dtype, E, K, Ds):
    H, D = (128, 256) if dtype == "bf16" else (64, 96)
    wl = mi.Workload("edge", "edge case", dtype, H, E, K, D, Ds, (1, 13, 130), 11, zipf_s=1.2)
    L = DeviceLayer(wl)
    for T in wl.Ts:
        run_and_check(M, L, T)


# CTA-pair layers (two reduction blocks per ring stage) whose second layer
# splits its reduction into an odd number of blocks per split (24 blocks as
# 5+5+5+5+4, or 24 over 5 at T = 384): the box of a split's last stage
# reaches into the next split's first block, which must not be multiplied.
@pytest.mark.parametrize("T,H,E,K,D,Ds", [(256, 768, 4, 2, 1536, 768), (384, 512, 4, 4, 1536, 512)])
def test_layer_pair_odd_blocks_per_split(M, T, H, E, K, D, Ds):
    wl = mi.Workload("pairsplit", "CTA pairs, odd reduction blocks per split", "bf16", H, E, K, D,
                     Ds, (T,), 23, zipf_s=0.8)
    run_and_check(M, DeviceLayer(wl), T)


def test_layer_empty_batch_is_a_no_op(M):
    L = layer("c1")
    d = L.desc(M, 0)
    ws = M.alloc_workspace(d)
    M.moe_layer_forward(d, L.weights(M), None, None, None, ws)
    torch.cuda.synchronize()


def test_workspace_too_small_is_rejected(M):
    L = layer("c1")
    d = L.desc(M, 64)
    small = torch.zeros(M.moe_workspace_size(d) - 256, dtype=torch.uint8, device="cuda")
    x = mi.draw_x(L.wl, 64).cuda()
    with pytest.raises(M.MoEError) as ei:
        M.moe_layer_forward(d, L.weights(M), x, torch.empty_like(x), None, small)
    assert ei.value.status == 3


# The benchmark times the expert GEMMs alone by re-running them on what the
# last forward left in the workspace (moe_expert_gemms): recomputing the same
# first-layer outputs and expert outputs must leave the workspace bit for bit
# as the forward left it, on CTA pairs (c2 T=512) and single-CTA tiles (c3 T=16).
@pytest.mark.parametrize("key,T", [("c2", 512), ("c3", 16)])
def test_expert_gemms_recompute_the_forward_bit_for_bit(M, key, T):
    L = layer(key)
    wl = L.wl
    x = mi.draw_x(wl, T).cuda()
    d = L.desc(M, T)
    ws = M.alloc_workspace(d)
    y = torch.empty_like(x)
    M.moe_layer_forward(d, L.weights(M), x, y, None, ws)
    torch.cuda.synchronize()
    before = ws.clone()
    M.moe_expert_gemms(d, L.weights(M), x, ws)
    torch.cuda.synchronize()
    assert M.moe_check_status(ws) == 0
    # (moe_check_status clears the status word, which was zero before)
    assert torch.equal(ws, before)
