#!/usr/bin/env python
"""MoE layer forward benchmark on B200: tokens/s and fraction of roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload c2] [--T 4096] [--no-sweep] [--no-cpu-baseline]

A step is one pass of the whole layer (router + selection, dispatch, grouped
expert FFN with the shared expert, combine) over one batch of T tokens of the
chosen workload (default: the Mixtral-shaped bf16 layer, H=4096, E=8, K=2,
D=14336, at T=4096). Inputs are seeded synthetic tensors resident in HBM
(1.9 GB of expert weights per step, larger than the 126 MB L2). Under
torchrun every rank runs an independent replica on its own token batch
(weak scaling, no data-path collective); timing is the max over ranks.

Rank 0 prints one JSON line. `--impl reference` times the fp64 CPU oracle on
a bounded sample of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import moe_inputs as mi  # noqa: E402

METRIC = "MoE layer tokens/s at 1 B200 + % of roofline (HBM GB/s decode, TFLOPS prefill)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
BAD_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default="c2")
    p.add_argument("--T", type=int, default=None)
    p.add_argument("--no-sweep", action="store_true", help="time the headline workload point only")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--sweep-only", default=None,
                   help="comma-separated workload keys the sweep covers (default: all)")
    p.add_argument("--cold-l2", action="store_true",
                   help="sweep points also report the median forward with L2 flushed before each call")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------- workload ---
def algorithmic(wl, T, touched, counts=None):
    """Algorithmic FLOPs and HBM bytes of one layer forward (and of the expert
    GEMMs alone). FLOPs: router 2*T*H*E, routed experts 4*T*K*H*D (2*H*D
    multiply-adds per copy, from the Kimi K3 page's Time_comp), shared expert
    4*T*H*Ds. Bytes: router weights, the weights of every expert the routing
    touched, the shared expert's weights, x in and y out."""
    es = 2 if wl.dtype == "bf16" else 4
    H, E, K, D, Ds = wl.H, wl.E, wl.K, wl.D, wl.Ds
    f_router = 2 * T * H * E
    f_gemm = 4 * T * K * H * D + 4 * T * H * Ds
    b_weights = touched * 2 * H * D * es + 2 * H * Ds * es
    b_layer = E * H * es + b_weights + 2 * T * H * es
    b_gemm = b_weights + T * H * es * (1 + (1 if Ds else 0)) + T * K * H * es
    return {"flops": f_router + f_gemm, "bytes": b_layer, "gemm_flops": f_gemm, "gemm_bytes": b_gemm}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the two
# expert-GEMM launches of one step, from one ncu capture of this workload
# (the committed ncu summary of the expert GEMM). Valid only for the kernel code
# it was measured on: the key is a fingerprint of the GEMM source and the
# headers it includes with comments and whitespace removed, so any change to
# the code (not to its comments) makes it null.
MEASURED_TRAFFIC = {"kernel_code_sha256_16": "847c8768f9eabbbe", "workload": "c2", "T": 4096,
                    "bytes_per_step": 1.106830e9 + 0.234959e9 + 1.445730e9 + 0.135528e9}
TRAFFIC_SOURCES = ("ffn_tc.cu", "common.cuh", "kernels.cuh")


def _strip_c_comments(text):
    """C/C++ source without comments or whitespace (string literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            if not c.isspace():
                out.append(c)
            i += 1
    return "".join(out)


def kernel_code_fingerprint():
    import hashlib
    h = hashlib.sha256()
    for name in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, "fine_grained_moe_router_b200", "csrc", name)) as f:
            h.update(_strip_c_comments(f.read()).encode())
    return h.hexdigest()[:16]


def measured_traffic(wl, T):
    m = MEASURED_TRAFFIC
    if (kernel_code_fingerprint() == m["kernel_code_sha256_16"] and wl.key == m["workload"]
            and T == m["T"]):
        return m["bytes_per_step"] / 2.0   # mean per launch of the two expert GEMMs
    return None


def roofline_bound(flops, nbytes, peaks):
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    return ("tensor", t_tc) if t_tc >= t_hbm else ("hbm", t_hbm)


# --------------------------------------------------------------- clocks ---
class ClockSampler:
    """SM clock and clock-event reasons of the benchmarked GPU during the timed
    region. Polls NVML from a thread every few milliseconds (a timed region
    of a few tens of milliseconds still gets samples); falls back to
    `nvidia-smi -lms 200` when NVML is not importable. Reads only."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, device: torch.device):
        self.device = device
        self.proc = None
        self.path = None
        self.thread = None
        self.samples = []
        self.max_mhz = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                u = str(uuid)
                return pynvml.nvmlDeviceGetHandleByUUID(u if u.startswith("GPU-") else "GPU-" + u)
            except Exception:
                pass
        bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
        return pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def start(self):
        import threading
        try:
            import pynvml
            h = self._nvml_handle()
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.stop_flag = threading.Event()

            def poll():
                while not self.stop_flag.is_set():
                    try:
                        mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                        rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((float(mhz), int(rs)))
                    except Exception:
                        pass
                    time.sleep(0.002)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            while not self.samples and self.thread.is_alive():   # first sample before timing
                time.sleep(0.001)
            return
        except Exception:
            self.thread = None
        try:
            scratch = os.path.join(ROOT, "_build")
            os.makedirs(scratch, exist_ok=True)
            fd, self.path = tempfile.mkstemp(suffix=".csv", dir=scratch)
            os.close(fd)
            idx = self.device.index if self.device.index is not None else 0
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(idx), "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            if not self.samples:
                return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"],
                        "source": "nvml"}
            reasons = sorted({n for _, r in self.samples for n, bit in self.REASONS if r & bit})
            return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                    "sm_max_mhz": self.max_mhz, "reasons": reasons,
                    "samples": len(self.samples), "source": "nvml"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for r in csv.reader(f):
                if len(r) >= 9:
                    rows.append([c.strip() for c in r])
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "source": "nvidia-smi"}


def build_and_import():
    """Builds libmoe.so if stale (by file path, before the package loads it)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_moe_build", os.path.join(ROOT, "fine_grained_moe_router_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import fine_grained_moe_router_b200 as M
    return M


# ------------------------------------------------------------ distributed ---
def dist_info():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------- CPU oracle ---
def oracle_inputs(wl, host, x):
    """fp64 widening of the inputs for the oracle (outside any timed region)."""
    return dict(x=mi.to_f64(x), wr=mi.to_f64(host["w_router"]), bias=host["bias"].numpy(),
                w1=mi.LazyF64(host["w1"]), w2=mi.LazyF64(host["w2"]),
                ws1=mi.to_f64(host["ws1"]), ws2=mi.to_f64(host["ws2"]))


def widen_all(inp):
    """Replace lazily widened expert weights by float64 arrays when memory allows."""
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = 0
    n = len(inp["w1"])
    need = 2 * n * inp["w1"].t[0].numel() * 8
    if avail > 3 * need:
        inp = dict(inp)
        inp["w1"] = [inp["w1"][e] for e in range(n)]
        inp["w2"] = [inp["w2"][e] for e in range(n)]
    return inp


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_size(wl, T):
    """Tokens whose expert FFNs the oracle computes per step: every token up to
    64, else the seeded sample the workloads name (128 tokens at the prefill
    scale, 64 otherwise). Routing and dispatch always cover all T tokens."""
    if T <= 64:
        return T
    return 128 if wl.key == "c5" else 64


def oracle_step(wl, inp, T, seed):
    """One step of the CPU baseline: routing and dispatch of all T tokens plus
    the expert FFNs and combine of a seeded token sample (fp64 oracle).
    Returns (seconds, tokens computed)."""
    import oracle
    tokens = mi.sample_tokens(T, oracle_sample_size(wl, T), seed).numpy()
    t0 = time.perf_counter()
    oracle.moe_layer_forward(inp["x"], inp["wr"], inp["bias"], inp["w1"], inp["w2"], inp["ws1"],
                             inp["ws2"], wl.K, tokens=tokens)
    return time.perf_counter() - t0, len(tokens)


def oracle_sample_text(wl, T, steps):
    return (f"{steps} steps, each: routing and dispatch of all {T} tokens + expert FFNs and "
            f"combine of {oracle_sample_size(wl, T)} seeded sample tokens (fp64 numpy oracle)")


# ------------------------------------------------------------ reference ---
def run_reference(args, wl, T):
    rank, world, _ = dist_info()
    if rank != 0:
        return
    host = mi.draw_layer(wl)
    x = mi.draw_x(wl, T)
    inp = widen_all(oracle_inputs(wl, host, x))
    for i in range(args.warmup):
        oracle_step(wl, inp, T, seed=100 + i)
    total, done = 0.0, 0
    for i in range(args.steps):
        dt, n = oracle_step(wl, inp, T, seed=200 + i)
        total += dt
        done += n
    value = done / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, T, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": oracle_sample_text(wl, T, args.steps)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(wl, T, world):
    return {"workload": f"{wl.name}: H={wl.H} E={wl.E} K={wl.K} D={wl.D} Ds={wl.Ds} T={T} ({wl.key})",
            "T": T, "H": wl.H, "E": wl.E, "K": wl.K, "D": wl.D, "Ds": wl.Ds,
            "global_batch": T * world, "l2": "inputs larger than L2 (expert weights "
            f"{2 * wl.E * wl.H * wl.D * (2 if wl.dtype == 'bf16' else 4) / 1e9:.2f} GB per step)",
            "parallelism": f"replicas x{world} (independent token batches, no collective)"}


# ----------------------------------------------------------------- ours ---
class Runner:
    def __init__(self, M, wl, dev, T, replica):
        self.M, self.wl, self.T = M, wl, T
        self.desc = M.make_desc(T, wl.H, wl.E, wl.K, wl.D, wl.Ds,
                                M.MOE_BF16 if wl.dtype == "bf16" else M.MOE_F32)
        self.dev = dev
        self.weights = M.make_weights(dev["w_router"], dev["w1"], dev["w2"], dev["ws1"], dev["ws2"],
                                      dev["bias"])
        self.ws = M.alloc_workspace(self.desc)
        self.x_host = mi.draw_x(wl, T, replica)
        self.x = self.x_host.cuda()
        self.y = torch.empty_like(self.x)
        self.counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
        self.routing = M.make_routing(counts=self.counts)

    def step(self):
        self.M.moe_layer_forward(self.desc, self.weights, self.x, self.y, self.routing, self.ws)

    def timed(self, steps, warmup, world, device, sampler=None):
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        if sampler is not None:
            sampler.start()   # clocks of the timed region only
        n0 = self.M.moe_kernel_launch_count()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(steps):
            self.step()
        end.record()
        torch.cuda.synchronize()
        launches = self.M.moe_kernel_launch_count() - n0
        if sampler is not None:
            self.clocks = sampler.stop()
        barrier(world)
        ms = max_over_ranks(start.elapsed_time(end), world, device)
        return ms, launches

    def timed_graph(self, steps, warmup):
        """The same forward captured once in a CUDA graph and replayed."""
        self.step()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.step()
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(steps):
            g.replay()
        end.record()
        torch.cuda.synchronize()
        del g
        return start.elapsed_time(end)

    def timed_cold(self, iters, warmup=3):
        """Median forward time (ms) with L2 flushed before every call: a buffer
        of twice the L2 size is written between calls, outside the events
        around the forward (both on the current stream)."""
        props = torch.cuda.get_device_properties(torch.cuda.current_device())
        l2 = int(getattr(props, "L2_cache_size", 0)) or (126 << 20)
        flush = torch.empty(2 * l2, dtype=torch.uint8, device="cuda")
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(iters)]
        for i in range(warmup + iters):
            flush.fill_(i & 0xFF)
            if i >= warmup:
                evs[i - warmup][0].record()
            self.step()
            if i >= warmup:
                evs[i - warmup][1].record()
        torch.cuda.synchronize()
        times = sorted(a.elapsed_time(b) for a, b in evs)
        del flush
        return times[len(times) // 2]

    def stages(self, steps):
        """Per-stage device times (ms, mean over steps) from events recorded
        between the kernels of moe_layer_forward_profiled."""
        M = self.M
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
        for s in range(steps):
            M.moe_layer_forward_profiled(self.desc, self.weights, self.x, self.y, self.routing, self.ws, evs[s])
        torch.cuda.synchronize()
        out = {}
        for i, name in enumerate(M.FORWARD_STAGES):
            out[name] = statistics.mean(evs[s][i].elapsed_time(evs[s][i + 1]) for s in range(steps))
        return out

    def e2e(self, steps, warmup, world, device):
        """Through the public API from pinned host memory: every step copies its
        x host -> device, runs the forward and copies its y device -> host, all
        inside the timed region. As a serving loop would, the copies run on a
        second stream with double-buffered device tensors, so step i+1's input
        copy and step i-1's output copy overlap step i's forward."""
        xh = self.x_host.pin_memory()
        yh = [torch.empty_like(xh).pin_memory() for _ in range(2)]
        xd = [self.x, torch.empty_like(self.x)]
        yd = [self.y, torch.empty_like(self.y)]
        comp = torch.cuda.current_stream()
        copy = torch.cuda.Stream()
        ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("h2d", "fwd", "d2h")}
        M = self.M

        def run(n, start=None):
            if start is not None:
                start.record(comp)
            copy.wait_stream(comp)
            with torch.cuda.stream(copy):
                xd[0].copy_(xh, non_blocking=True)
                ev["h2d"][0].record(copy)
            for i in range(n):
                b = i % 2
                comp.wait_event(ev["h2d"][b])
                if i >= 2:
                    comp.wait_event(ev["d2h"][b])        # y buffer b has left for the host
                M.moe_layer_forward(self.desc, self.weights, xd[b], yd[b], self.routing, self.ws,
                                    comp)
                ev["fwd"][b].record(comp)
                with torch.cuda.stream(copy):
                    if i + 1 < n:
                        nb = (i + 1) % 2
                        if i >= 1:
                            copy.wait_event(ev["fwd"][nb])   # x buffer nb is no longer read
                        xd[nb].copy_(xh, non_blocking=True)
                        ev["h2d"][nb].record(copy)
                    copy.wait_event(ev["fwd"][b])
                    yh[b].copy_(yd[b], non_blocking=True)
                    ev["d2h"][b].record(copy)
            comp.wait_stream(copy)

        run(warmup)
        torch.cuda.synchronize()
        barrier(world)
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        run(steps, start)
        end.record(comp)
        torch.cuda.synchronize()
        barrier(world)
        ms = max_over_ranks(start.elapsed_time(end), world, device)
        nbytes = xh.numel() * xh.element_size()
        return ms, nbytes, yh[0].numel() * yh[0].element_size()

    def timed_gemms(self, steps, warmup=3):
        """Device time (ms) per pair of the step's two expert-GEMM launches, run
        again back to back (moe_expert_gemms) on the dispatched rows and tile
        lists the last forward left in the workspace; CUDA events on the
        launching stream. None where the layer runs as a single launch."""
        M = self.M
        self.step()
        try:
            for _ in range(warmup):
                M.moe_expert_gemms(self.desc, self.weights, self.x, self.ws)
        except M.MoEError:
            return None
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(steps):
            M.moe_expert_gemms(self.desc, self.weights, self.x, self.ws)
        end.record()
        torch.cuda.synchronize()
        return start.elapsed_time(end) / steps

    def touched(self):
        return int((self.counts > 0).sum().item())


def gemm_roofline(R, wl, T, alg, peaks, steps, ms_step):
    """Roofline of the dominant kernels: the two grouped expert-GEMM launches,
    timed as a pair in a loop of their own (Runner.timed_gemms). Achieved =
    the GEMMs' algorithmic FLOPs (tensor-bound) or bytes (HBM-bound) per pair
    / the measured time per pair. Where the whole layer is one launch, the
    dominant kernel is that launch and the step time is its time."""
    gemm_ms = R.timed_gemms(steps)
    single = gemm_ms is None
    if single:
        bound, _ = roofline_bound(alg["flops"], alg["bytes"], peaks)
        flops, nbytes, t_ms = alg["flops"], alg["bytes"], ms_step
        kernel = "single-launch decode forward (router, dispatch, expert GEMVs, combine)"
    else:
        bound, _ = roofline_bound(alg["gemm_flops"], alg["gemm_bytes"], peaks)
        flops, nbytes, t_ms = alg["gemm_flops"], alg["gemm_bytes"], gemm_ms
        kernel = "grouped expert GEMMs (GEMM1 + GeLU, GEMM2; shared expert included)"
    if bound == "tensor":
        achieved, peak, unit = flops / (t_ms / 1e3) / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    else:
        achieved, peak, unit = nbytes / (t_ms / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s"
    out = {"kernel": kernel, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
           "frac": achieved / peak,
           # the same against the seconds-long (power-capped) GEMM figure
           "frac_of_sustained": (achieved / peaks["bf16_tflops_sustained"]
                                 if bound == "tensor" else None),
           "ms_per_launch_pair": None if single else gemm_ms,
           "share_of_step": 1.0 if single else gemm_ms / ms_step,
           # the kernels' own time cannot exceed the step that contains them
           "within_step": True if single else gemm_ms <= ms_step * 1.001}
    return out


def run_ours(args, wl, T):
    rank, world, local = dist_info()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    M = build_and_import()
    peaks, peaks_src = load_peaks()

    host = mi.draw_layer(wl)
    dev = {k: (v.to(device) if v is not None else None) for k, v in host.items()}
    R = Runner(M, wl, dev, T, replica=rank)

    ms, launches = R.timed(args.steps, args.warmup, world, device, sampler=ClockSampler(device))
    clocks = R.clocks
    ms_step = ms / args.steps
    value = world * T * args.steps / (ms / 1e3)

    stages = R.stages(args.steps)
    touched = R.touched()
    alg = algorithmic(wl, T, touched)
    rl = gemm_roofline(R, wl, T, alg, peaks, args.steps, ms_step)
    lbound, t_roof = roofline_bound(alg["flops"], alg["bytes"], peaks)

    e2e_ms, h2d, d2h = R.e2e(args.steps, args.warmup, world, device)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded: x ~ N(0,1), weights ~ N(0,1/fan_in) in bf16, Zipf logit skew "
                "as a bias input where the workload has one)",
        "config": workload_config(wl, T, world),
        "roofline": dict(rl, traffic=measured_traffic(wl, T),
                         traffic_unit="DRAM bytes per launch (mean of GEMM1 and GEMM2)",
                         peak_source=peaks_src),
        "layer_roofline": {"bound": lbound, "t_roof_ms": 1e3 * t_roof, "frac": 1e3 * t_roof / ms_step,
                           "flops": alg["flops"], "bytes": alg["bytes"], "experts_touched": touched},
        "stages_ms": stages,
        "e2e": {"value": world * T * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if not args.no_sweep and world == 1:
        only = args.sweep_only.split(",") if args.sweep_only else None
        line["sweep"] = sweep(M, wl, dev, T, peaks, only, args.cold_l2)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, host, R.x_host, T)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def measure_point(M, wl, dev, T, peaks, steps=20, warmup=5, cold=False):
    R = Runner(M, wl, dev, T, replica=0)
    ms, _ = R.timed(steps, warmup, 1, None)
    st = R.stages(steps)
    alg = algorithmic(wl, T, R.touched())
    bound, t_roof = roofline_bound(alg["flops"], alg["bytes"], peaks)
    ms_step = ms / steps
    graph_ms = R.timed_graph(steps, warmup) / steps
    rl = gemm_roofline(R, wl, T, alg, peaks, steps, ms_step)
    out = {"workload": wl.key, "T": T, "tokens_per_s": T / (ms_step / 1e3), "us_per_step": 1e3 * ms_step,
           "graph_us_per_step": 1e3 * graph_ms, "graph_frac": 1e3 * t_roof / graph_ms,
           "bound": bound, "roofline_us": 1e6 * t_roof, "frac": 1e3 * t_roof / ms_step,
           "experts_touched": R.touched(),
           "dominant": {"kernel": rl["kernel"], "bound": rl["bound"], "achieved": rl["achieved"],
                        "unit": rl["unit"], "frac": rl["frac"],
                        "us_per_launch_pair": (None if rl["ms_per_launch_pair"] is None
                                               else 1e3 * rl["ms_per_launch_pair"]),
                        "within_step": rl["within_step"]},
           "stages_us": {k: 1e3 * v for k, v in st.items()}}
    if cold:
        cold_ms = R.timed_cold(max(steps, 50))
        out["cold_l2_us_per_step"] = 1e3 * cold_ms
        out["cold_l2_frac"] = 1e3 * t_roof / cold_ms
    return out


def sweep(M, wl, dev, T_main, peaks, only=None, cold=False):
    """Every point of every workload (the headline point excepted), each
    workload's weights resident only while its points run."""
    keys = ["c1", "c2", "c3", "c4", "c5"] if not only else only
    out = []
    for key in keys:
        w2 = mi.WORKLOADS[key]
        if key == wl.key:
            d2 = dev
        else:
            host = mi.draw_layer(w2)
            d2 = {k: (v.cuda() if v is not None else None) for k, v in host.items()}
            del host
        for T in w2.Ts:
            if key == wl.key and T == T_main:
                continue
            out.append(measure_point(M, w2, d2, T, peaks, cold=cold))
        if key != wl.key:
            del d2
            torch.cuda.empty_cache()
    return out


def cpu_baseline(wl, host, x, T, target_s=12.0):
    """The oracle on the host cores, with the reference arm's per-step program
    (oracle_step), repeated until about target_s seconds of CPU work."""
    inp = widen_all(oracle_inputs(wl, host, x))
    oracle_step(wl, inp, T, seed=99)          # warm-up (first touch of the weights)
    total, done, steps = 0.0, 0, 0
    while steps < 1 or total < target_s:
        dt, n = oracle_step(wl, inp, T, seed=300 + steps)
        total += dt
        done += n
        steps += 1
    return {"value": done / total, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": oracle_sample_text(wl, T, steps) + f", {total:.1f} s"}


def main():
    args = parse_args()
    wl = mi.WORKLOADS[args.workload]
    T = args.T if args.T is not None else max(wl.Ts)
    if args.impl == "reference":
        run_reference(args, wl, T)
    else:
        run_ours(args, wl, T)


if __name__ == "__main__":
    main()
