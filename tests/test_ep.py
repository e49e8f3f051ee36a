"""Expert-parallel forward (fine_grained_moe_router_b200.ep) on CPU ranks.

Two (and one) gloo ranks run ExpertParallelMoE's exchange logic -- counts
All-to-All, dispatched rows out, expert outputs back, local expert-major
order -- with the compute steps done by a stand-in built from the fp64 oracle
(no GPU here). Every rank's output must equal the oracle's single-process
forward of the whole batch on that rank's tokens ("Kimi K3 fine-grained MoE
under high concurrency", section "物理通信拓扑": dispatch All-to-All, local
experts, combine All-to-All). The CUDA path of the same class runs in
tests/test_gpu_ep.py.
"""
import json
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

H, E, K, D, DS = 16, 8, 2, 24, 12
T_OF_RANK = (13, 7, 0, 5)   # one rank with no tokens at all


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def layer_weights(seed=5):
    g = np.random.default_rng(seed)
    return dict(wr=g.normal(size=(E, H)) / math.sqrt(H), w1=g.normal(size=(E, D, H)) / math.sqrt(H),
                w2=g.normal(size=(E, H, D)) / math.sqrt(D), ws1=g.normal(size=(DS, H)) / math.sqrt(H),
                ws2=g.normal(size=(H, DS)) / math.sqrt(DS), bias=g.uniform(-0.3, 0.3, size=E))


def tokens_of(rank, seed=7):
    return np.random.default_rng(seed + rank).normal(size=(T_OF_RANK[rank], H))


def local_order_reference(recv_counts):
    """The expert-major order of the received rows, from its definition."""
    c = np.asarray(recv_counts, np.int64)
    G, El = c.shape
    src_start = np.cumsum(c.reshape(-1)) - c.reshape(-1)        # source-major layout
    order = []
    for e in range(El):
        for s in range(G):
            start = src_start[s * El + e]
            order.extend(range(start, start + c[s, e]))
    perm = np.array(order, dtype=np.int64)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    off = np.concatenate([[0], np.cumsum(c.sum(axis=0))])
    return off, perm, inv


class OracleOps:
    """fp64 stand-ins for the compute steps (test only)."""

    def __init__(self):
        sys.path.insert(0, ROOT)
        import oracle
        self.o = oracle

    def route(self, x, w_router, bias, K_, cf):
        logits = self.o.router_logits(x.numpy(), w_router.numpy())
        idx, w, _ = self.o.select_topk(logits, None if bias is None else bias.numpy(), K_)
        return torch.from_numpy(logits), torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(w)

    def dispatch(self, idx, E_):
        c, off, perm, inv = self.o.dispatch(idx.numpy(), E_)
        return tuple(torch.from_numpy(np.asarray(a, np.int32)) for a in (c, off, perm, inv))

    def gather_rows(self, src, idx, divisor):
        return src[idx.long() // divisor].clone()

    def local_order(self, recv_counts):
        off, perm, inv = local_order_reference(recv_counts.numpy())
        return tuple(torch.from_numpy(a.astype(np.int32)) for a in (off, perm, inv))

    def experts(self, rows, perm, offsets, w1, w2):
        y, _ = self.o.grouped_ffn(rows.numpy(), perm.numpy(), offsets.numpy(), 1, w1.numpy(),
                                  w2.numpy())
        return torch.from_numpy(y)

    def combine(self, y_rows, topk_w, inv, y_shared, out_dtype):
        y = self.o.combine(y_rows.numpy(), topk_w.numpy(), inv.numpy(),
                           None if y_shared is None else y_shared.numpy())
        return torch.from_numpy(y)


def _rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    from fine_grained_moe_router_b200.ep import ExpertParallelMoE
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        W = layer_weights()
        El = E // world
        t = {k: torch.from_numpy(v) for k, v in W.items()}
        layer = ExpertParallelMoE(t["wr"], t["w1"][rank * El:(rank + 1) * El],
                                  t["w2"][rank * El:(rank + 1) * El], K, t["ws1"], t["ws2"],
                                  t["bias"], ops=OracleOps())
        routing = {}
        y = layer(torch.from_numpy(tokens_of(rank)), routing=routing)
        res = {"y": y.numpy().tolist(), "recv": routing["recv_counts"].numpy().tolist()}
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


@pytest.mark.parametrize("world", [1, 2, 4])
def test_expert_parallel_forward_equals_single_process_oracle(tmp_path, world):
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    sys.path.insert(0, ROOT)
    import oracle
    W = layer_weights()
    xs = [tokens_of(r) for r in range(world)]
    ref = oracle.moe_layer_forward(np.concatenate(xs), W["wr"], W["bias"], W["w1"], W["w2"],
                                   W["ws1"], W["ws2"], K)
    El = E // world
    counts = np.asarray(ref["counts"]).reshape(world, El)   # row g: the experts rank g owns
    start = 0
    for r in range(world):
        res = json.load(open(tmp_path / f"rank{r}.json"))
        y = np.asarray(res["y"]).reshape(-1, H)
        np.testing.assert_allclose(y, ref["y"][start:start + xs[r].shape[0]], rtol=1e-12,
                                   atol=1e-12)
        start += xs[r].shape[0]
        # the owner received every copy of each of its experts exactly once
        recv = np.asarray(res["recv"]).reshape(world, El)
        np.testing.assert_array_equal(recv.sum(axis=0), counts[r])


def test_local_order_reference_definition():
    # two sources, three local experts: rows arrive source-major, each source's by expert
    c = np.array([[2, 0, 1], [1, 3, 0]])
    off, perm, inv = local_order_reference(c)
    assert off.tolist() == [0, 3, 6, 7]
    # receive positions: s0: e0 -> 0,1; e2 -> 2; s1: e0 -> 3; e1 -> 4,5,6
    assert perm.tolist() == [0, 1, 3, 4, 5, 6, 2]
    assert (perm[inv] == np.arange(7)).all()
