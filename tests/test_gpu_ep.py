"""The expert-parallel pieces on the GPU: the expert-major order of received
rows (moe_ep_local_order) and the row gather (moe_gather_rows) against their
definitions, and ExpertParallelMoE through its CUDA path on one NCCL rank
against the oracle (the exchanges then move every row to the same rank; the
CPU tests in tests/test_ep.py run the exchange logic on 2 and 4 ranks)."""
import socket

import numpy as np
import pytest
import torch

import moe_inputs as mi
from parity import DeviceLayer, check_layer, to_np
from test_ep import local_order_reference

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    from _lib import build_and_import
    return build_and_import()


@pytest.mark.parametrize("G,El,hi", [(1, 1, 5), (2, 3, 4), (4, 16, 9), (8, 512, 3), (3, 64, 0)])
def test_local_order_matches_definition(M, G, El, hi):
    rng = np.random.default_rng(G * 100 + El)
    c = rng.integers(0, hi + 1, size=(G, El)).astype(np.int32)
    off, perm, inv = local_order_reference(c)
    R = int(c.sum())
    d_off = torch.full((El + 1,), -7, dtype=torch.int32, device="cuda")
    d_perm = torch.full((R,), -7, dtype=torch.int32, device="cuda")
    d_inv = torch.full((R,), -7, dtype=torch.int32, device="cuda")
    M.moe_ep_local_order(torch.from_numpy(c).cuda(), d_off, d_perm, d_inv)
    torch.cuda.synchronize()
    assert (to_np(d_off) == off).all()
    assert (to_np(d_perm) == perm).all() and (to_np(d_inv) == inv).all()


@pytest.mark.parametrize("dtype,cols", [(torch.bfloat16, 4096), (torch.float32, 4096),
                                        (torch.bfloat16, 8)])
def test_gather_rows_matches_indexing(M, dtype, cols):
    rng = np.random.default_rng(cols)
    src = torch.randn(300, cols, dtype=torch.float32).to(dtype).cuda()
    div = 3
    idx = rng.integers(0, 300 * div, size=500).astype(np.int32)
    idx[::17] = 300 * div + 5                      # out of range: row left unwritten
    dst = torch.full((500, cols), 7.0, dtype=dtype, device="cuda")
    M.moe_gather_rows(src, torch.from_numpy(idx).cuda(), div, dst)
    torch.cuda.synchronize()
    want = src.cpu()[np.minimum(idx // div, 299)]
    ok = idx < 300 * div
    assert torch.equal(dst.cpu()[ok], want[ok])
    assert (dst.cpu()[~ok] == 7.0).all()


def test_expert_parallel_forward_on_one_nccl_rank(M):
    import torch.distributed as dist
    from fine_grained_moe_router_b200.ep import ExpertParallelMoE
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        wl = mi.with_shape(mi.WORKLOADS["c3"], H=512, D=256, Ds=512)
        L = DeviceLayer(wl)
        dv = L.dev
        layer = ExpertParallelMoE(dv["w_router"], dv["w1"], dv["w2"], wl.K, dv["ws1"], dv["ws2"],
                                  dv["bias"])
        for T in (1, 37, 300):
            x = mi.draw_x(wl, T)
            routing = {}
            y = layer(x.cuda(), routing=routing)
            torch.cuda.synchronize()
            g = {"logits": to_np(routing["logits"]), "topk_idx": to_np(routing["topk_idx"]),
                 "topk_w": to_np(routing["topk_w"]), "counts": to_np(routing["counts"])}
            check_layer(wl, x, L, g, to_np(y))
            assert (to_np(routing["recv_counts"]).reshape(-1) == g["counts"]).all()
    finally:
        dist.destroy_process_group()
