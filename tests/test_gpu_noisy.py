"""Gumbel-noise routing ("MoE architecture in production" §2.3) on the GPU
against the oracle: selection from given logits and noise bit for bit, and
the whole noisy layer forward within the layer tolerances."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from parity import DeviceLayer, W_TOL, check_layer, routing_buffers, routing_np, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    from _lib import build_and_import
    return build_and_import()


@pytest.mark.parametrize("T,E,K,ties", [(1, 8, 2, False), (37, 16, 3, True), (300, 128, 8, False),
                                        (129, 512, 16, True), (64, 256, 8, False)])
def test_noisy_topk_from_logits_bit_exact(M, T, E, K, ties):
    rng = np.random.default_rng(T * 7 + E)
    if ties:
        vals = np.array([-1.0, 0.0, 0.5, 0.5, 1.0], np.float32)
        logits = rng.choice(vals, size=(T, E)).astype(np.float32)
        g = rng.choice(np.array([-0.5, 0.0, 0.5], np.float32), size=(T, E))   # ties survive
    else:
        logits = rng.normal(size=(T, E)).astype(np.float32)
        g = mi.draw_gumbel(T, E, seed=T + E).numpy()
    b = rng.uniform(-0.5, 0.5, size=E).astype(np.float32)
    d = M.make_desc(T, 256, E, K, 256, 0, M.MOE_F32)
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    M.moe_topk_from_logits_noisy(d, torch.from_numpy(logits).cuda(), torch.from_numpy(b).cuda(),
                                 torch.from_numpy(g).cuda(), idx, w)
    ref_idx, ref_w, _ = oracle.select_topk(logits.astype(np.float64), b, K, noise=g)
    assert (to_np(idx) == ref_idx).all()
    assert np.max(np.abs(to_np(w) - ref_w)) <= W_TOL


@pytest.mark.parametrize("key,shape,T", [("c3", dict(H=512, D=256, Ds=512), 16),
                                         ("c4", dict(H=512, D=256, Ds=512), 200),
                                         ("c1", {}, 64)])
def test_noisy_layer_matches_oracle(M, key, shape, T):
    wl = mi.with_shape(mi.WORKLOADS[key], **shape)
    L = DeviceLayer(wl)
    d = L.desc(M, T)
    x = mi.draw_x(wl, T)
    g = mi.draw_gumbel(T, wl.E, seed=wl.seed + T)
    xd = x.cuda()
    y = torch.full_like(xd, float("nan"))
    r = routing_buffers(wl, T)
    ws = M.alloc_workspace(d)
    M.moe_layer_forward_noisy(d, L.weights(M), xd, g.cuda(), y, M.make_routing(**r), ws)
    torch.cuda.synchronize()
    assert M.moe_check_status(ws) == 0
    gn = g.numpy()
    # the oracle is routed from the GPU's logits with the same noise
    ref = check_layer(wl, x, L, routing_np(r), to_np(y), noise=gn)
    # the noise changes the routing of some tokens
    plain_idx, _, _ = oracle.select_topk(ref["logits"], L.bias, wl.K)
    assert (plain_idx != ref["idx"]).any()


def test_zero_noise_equals_plain_forward(M):
    wl = mi.with_shape(mi.WORKLOADS["c3"], H=256, D=128, Ds=256)
    L = DeviceLayer(wl)
    T = 40
    d = L.desc(M, T)
    xd = mi.draw_x(wl, T).cuda()
    ws = M.alloc_workspace(d)
    y0, y1 = torch.empty_like(xd), torch.empty_like(xd)
    M.moe_layer_forward(d, L.weights(M), xd, y0, None, ws)
    M.moe_layer_forward_noisy(d, L.weights(M), xd, torch.zeros((T, wl.E), device="cuda"), y1, None, ws)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
