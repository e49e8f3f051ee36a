"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, as torchrun would
launch them. Checks the max-over-ranks reduction of the timing, the barrier,
and that only rank 0 of the reference arm works and prints."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, w, local = bench.dist_info()
        res = {"rank": r, "world": w, "local": local}
        # each rank reports a different device time; every rank must get the max
        res["max"] = bench.max_over_ranks(1.5 + rank, w, "cpu")
        bench.barrier(w)
        # reference arm: rank 0 times the oracle and prints one line, the others return
        wl = bench.mi.with_shape(bench.mi.WORKLOADS["c1"], H=64, D=96, E=4, K=2)
        ns = type("A", (), {"steps": 1, "warmup": 0, "gpus": w})()
        buf = io.StringIO()
        with redirect_stdout(buf):
            bench.run_reference(ns, wl, 8)
        res["printed"] = buf.getvalue()
        bench.barrier(w)
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, x in enumerate(res):
        assert (x["rank"], x["world"], x["local"]) == (r, world, r)
        assert x["max"] == pytest.approx(1.5 + world - 1)
    line = json.loads(res[0]["printed"].strip())
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["global_batch"] == 8 * world
    assert res[1]["printed"] == ""
