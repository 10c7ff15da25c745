#!/usr/bin/env python3
"""Benchmark of the MoE expert layer (route -> permute -> int4 grouped GEMMs
with SwiGLU -> combine) through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One step = one strata_moe_forward over one batch of the workload (default:
the 6144-token prefill chunk, d=4096, 512 experts, top-10, n=1024, int4 with
group 64).  Inputs are seeded synthetic tensors resident in HBM; the weights
(3.4 GB) exceed the 126 MB L2, so no flush is needed between steps.  Prints one
JSON line.  With N > 1 (torchrun), every rank runs an independent replica
(the layer shards by token batches with no exchange); the time is the max over
ranks and `value` the total tokens of all ranks per second.

--impl reference times the fp64 CPU oracle on a bounded token sample of the
same workload on the host cores (rank 0 only).
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "MoE-layer tokens/s at T=6144, 512 experts top-10; % of tensor/HBM roofline"
# Sources each profiled kernel is built from: its DRAM counters in
# profiles/traffic.json stand only while these files are unchanged.
KERNEL_SOURCES = {
    "gemm_gate_up_large": ["local_moe_route_b200/csrc/gemm_tc.cu",
                           "local_moe_route_b200/csrc/common.cuh"],
    "gemm_gate_up_verify4": ["local_moe_route_b200/csrc/gemm_decode.cu",
                             "local_moe_route_b200/csrc/common.cuh"],
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        return self.summarise(self.lines)

    @staticmethod
    def summarise(lines):
        """Median SM clock under load, the maximum clock and the throttle
        reasons seen active, from nvidia-smi CSV lines in FIELDS order."""
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        busy = [v for v in sm if mx and v > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- model
def device_layer(inp, dev):
    import torch
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    L = {"x": t(inp["x"]).view(torch.bfloat16), "w_router": t(inp["w_router"]).view(torch.bfloat16),
         "bias": None if inp.get("bias") is None else t(inp["bias"])}
    for n in ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s"):
        L[n] = t(inp[n])
    return L


def launches_per_step(T, d, E):
    """Kernel launches of one strata_moe_forward (mirrors the dispatch rules)."""
    n = 2                    # router logits + top-k/softmax
    tc_router = T >= 128 and E % 128 == 0
    if not tc_router and T <= 16 and d // 32 > 1:
        n += 1               # sum of the K-split partial logits
    n += 3                   # permutation: histogram, scan, scatter
    n += 1                   # expert work lists
    n += 2 if T > 8 else 1   # gate/up (+ fp16 copy of x on the tensor-core path)
    n += 1                   # down
    n += 1                   # combine
    return n


def kernel_source_hash(kernel):
    h = hashlib.sha256()
    for p in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def profiled_traffic(kernel):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(kernel)
    if not e or kernel not in KERNEL_SOURCES or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------- ranks
def max_over_ranks(v, device=None):
    """Maximum of a per-rank float over all ranks (identity without a process
    group).  The timed region's duration is taken this way."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(v)
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, world, max_ms):
    """Whole-job tokens/s: tokens of all ranks over the slowest rank's time."""
    return tokens_per_rank * world / (max_ms / 1e3)


# --------------------------------------------------------------------------- our arm
def run_ours(args, wl):
    import torch
    import torch.distributed as dist
    import local_moe_route_b200 as sm

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=300))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    sm.lib()                                       # fails loudly without the library

    inp = make_inputs(wl)
    L = device_layer(inp, dev)
    dims = wl.dims()
    T, d, k, n, E = wl.T, wl.d, wl.k, wl.n, wl.E
    S = T * k
    ws = sm.workspace(dims, dev)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    gate, up, down = (L["gate_q"], L["gate_s"]), (L["up_q"], L["up_s"]), (L["down_q"], L["down_s"])
    stream = torch.cuda.current_stream()

    def forward(x=None, out=None):
        st = sm.strata_moe_forward(L["x"] if x is None else x, L["w_router"], L["bias"], gate, up,
                                   down, dims, y if out is None else out, None, None, ws,
                                   stream=torch.cuda.current_stream())
        if st != sm.STRATA_OK:
            raise sm.StrataError(st, "forward")

    # Small batches (decode / verify) replay the forward as one CUDA graph:
    # ten short kernels would otherwise wait on host launch overhead.  Large
    # batches launch eagerly (the GPU is the bottleneck there).
    graph = None
    if T <= 64:
        forward()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            forward()
        torch.cuda.synchronize()
    step = graph.replay if graph is not None else forward
    # weights a small batch touches can fit in L2; those runs flush it
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev) if T <= 64 else None

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- headline: K forwards, device time
    for _ in range(args.warmup):
        step()
    clocks = ClockSampler(dev.index) if rank == 0 else None
    barrier()
    if clocks:
        clocks.start()
        time.sleep(0.3)
    if flush is None:
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        ev0.record(stream)
        step_ev[0].record(stream)
        for i in range(args.steps):
            step()
            step_ev[i + 1].record(stream)
        ev1.record(stream)
        barrier()
        step_ms = [step_ev[i].elapsed_time(step_ev[i + 1]) for i in range(args.steps)]
        total_ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
    else:
        # the touched weights would stay in L2 from one step to the next:
        # overwrite L2 between steps and time each step alone
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        for a_, b_ in pairs:
            flush.zero_()
            a_.record(stream)
            step()
            b_.record(stream)
        barrier()
        step_ms = [a_.elapsed_time(b_) for a_, b_ in pairs]
        total_ms = max_over_ranks(sum(step_ms), dev)
    clk = clocks.stop() if clocks else None
    assert sm.strata_moe_device_status(stream) == sm.STRATA_OK

    if args.only_forward:
        if world > 1:
            dist.destroy_process_group()
        if rank != 0:
            return None
        return {"config": {"workload": wl.name}, "ms_per_step": round(total_ms / args.steps, 4),
                "value": round(job_throughput(T * args.steps, world, total_ms), 1),
                "unit": "tokens/s",
                "note": "forward only (profiling run)"}

    # ---- breakdown: the same layer as separate entry points, events around each
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    wts = torch.empty((T, k), dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    st_ = torch.empty(S, dtype=torch.int32, device=dev)
    sr_ = torch.empty(S, dtype=torch.int32, device=dev)
    h = torch.empty((S, n), dtype=torch.float16, device=dev)
    rows = torch.empty((S, d), dtype=torch.float16, device=dev)
    names = ["route", "permute", "gate_up", "down", "combine"]

    def staged(evs):
        evs[0].record(stream)
        sm.check(sm.strata_moe_route(L["x"], L["w_router"], L["bias"], dims, ids, wts, None, ws,
                                     stream=stream))
        evs[1].record(stream)
        sm.check(sm.strata_moe_permute(ids, dims, counts, offsets, st_, sr_, ws, stream=stream))
        evs[2].record(stream)
        sm.check(sm.strata_moe_expert_gemm_q4(sm.STRATA_OP_GATE_UP_SWIGLU, L["x"], st_, offsets,
                                              gate, up, None, dims, h, ws, stream=stream))
        evs[3].record(stream)
        sm.check(sm.strata_moe_expert_gemm_q4(sm.STRATA_OP_DOWN, h, None, offsets, down, None,
                                              None, dims, rows, ws, stream=stream))
        evs[4].record(stream)
        sm.check(sm.strata_moe_combine(rows, wts, sr_, dims, y, stream=stream))
        evs[5].record(stream)

    for _ in range(max(1, args.warmup)):
        staged([torch.cuda.Event(enable_timing=True) for _ in range(6)])
    barrier()
    per = {nm: [] for nm in names}
    for _ in range(args.steps):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        staged(evs)
        torch.cuda.synchronize()
        for i, nm in enumerate(names):
            per[nm].append(evs[i].elapsed_time(evs[i + 1]))
    stage_ms = {nm: statistics.mean(v) for nm, v in per.items()}

    # ---- end to end: host x -> device, forward, y -> host, every step
    x_host = torch.from_numpy(inp["x"]).view(torch.bfloat16).pin_memory()
    if flush is not None:
        # small batches: one step at a time, L2 flushed before each, each
        # step (copy in, forward, copy out) timed alone
        y_host = torch.empty((T, d), dtype=torch.bfloat16).pin_memory()
        x_dev = torch.empty_like(L["x"])
        for _ in range(args.warmup):
            x_dev.copy_(x_host, non_blocking=True)
            forward(x_dev)
            y_host.copy_(y, non_blocking=True)
        barrier()
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        for a_, b_ in pairs:
            flush.zero_()
            a_.record(stream)
            x_dev.copy_(x_host, non_blocking=True)
            forward(x_dev)
            y_host.copy_(y, non_blocking=True)
            b_.record(stream)
        barrier()
        e2e_elapsed = sum(a_.elapsed_time(b_) for a_, b_ in pairs)
    else:
        # large batches: copies pipelined against compute.  Step i's input is
        # copied in on one stream and its output copied out on another while
        # the forward of the neighbouring step runs; two device buffers each.
        y_host = [torch.empty((T, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        x_dev = [torch.empty_like(L["x"]) for _ in range(2)]
        y_dev = [torch.empty_like(y) for _ in range(2)]
        h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        x_free = [ev(), ev()]      # forward that read x_dev[b] is done
        y_free = [ev(), ev()]      # copy-out of y_dev[b] is done
        for b_ in range(2):
            x_free[b_].record(stream)
            y_free[b_].record(stream)

        def e2e_step(i):
            b_ = i & 1
            x_in, fwd_done = ev(), ev()
            with torch.cuda.stream(h2d):
                h2d.wait_event(x_free[b_])
                x_dev[b_].copy_(x_host, non_blocking=True)
                x_in.record(h2d)
            stream.wait_event(x_in)
            stream.wait_event(y_free[b_])
            forward(x_dev[b_], out=y_dev[b_])
            fwd_done.record(stream)
            x_free[b_].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(fwd_done)
                y_host[b_].copy_(y_dev[b_], non_blocking=True)
                y_free[b_].record(d2h)

        for i in range(args.warmup):
            e2e_step(i)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            e2e_step(i)
        stream.wait_event(y_free[0])
        stream.wait_event(y_free[1])
        e1.record(stream)
        barrier()
        e2e_elapsed = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_elapsed, dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    hbm, tf_burst, tf_sus, peak_kind = measured_peaks()
    tokens = T * args.steps * world
    value = job_throughput(T * args.steps, world, total_ms)
    ms_step = total_ms / args.steps
    tensor_bound = T > 8
    if tensor_bound:
        # dominant kernel: gate/up grouped GEMM; algorithmic FLOPs per launch
        flops = 2.0 * S * 2 * d * n
        dur = stage_ms["gate_up"] / 1e3
        achieved = flops / dur / 1e12
        roof = {"bound": "tensor",
                "kernel": "gate/up step: work lists + grouped fp16 copy of x + "
                          "moe_gemm_q4_tc_kernel<0,0> (gate/up + SwiGLU), one entry-point call",
                "achieved": round(achieved, 1), "peak": tf_burst, "unit": "TFLOP/s",
                "frac": round(achieved / tf_burst, 4),
                "peak_kind": f"{peak_kind} bf16 dense burst (fp16 dense is the same rate)",
                "algorithmic_per_launch": flops,
                "traffic": profiled_traffic("gemm_gate_up_" + wl.name)}
    else:
        ids_np = ids.cpu().numpy()
        touched = len(np.unique(ids_np))
        per_expert = (2 * n * d // 2 + 2 * n * (d // wl.group) * 2 + d * n // 2 + d * (n // wl.group) * 2)
        bytes_ = touched * per_expert * 2 / 3        # gate+up share of the touched experts
        dur = stage_ms["gate_up"] / 1e3
        achieved = bytes_ / dur / 1e9
        roof = {"bound": "hbm",
                "kernel": "gate/up step: work lists + moe_gemm_q4_decode_kernel<2, G> "
                          "(gate/up + SwiGLU), one entry-point call",
                "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "peak_kind": f"{peak_kind} copy bandwidth",
                "algorithmic_per_launch": bytes_,
                "traffic": profiled_traffic("gemm_gate_up_" + wl.name)}
    layer_flops = 2.0 * S * 3 * d * n + 2.0 * T * d * E
    layer_roof = None
    if not tensor_bound:
        # the whole layer against HBM: weights of the experts the batch touches,
        # the router matrix, x and y, over the step time
        per_exp = 3 * n * d // 2 + 3 * n * (d // wl.group) * 2
        lbytes = touched * per_exp + d * E * 2 + 2 * T * d * 2
        lach = lbytes / (ms_step / 1e3) / 1e9
        layer_roof = {"bound": "hbm", "achieved": round(lach, 1), "peak": hbm, "unit": "GB/s",
                      "frac": round(lach / hbm, 4), "bytes_per_step": lbytes,
                      "experts_touched": touched}
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int4xfp16",
        "data": "synthetic (seeded, shapes of the pages' workload)",
        "config": {"workload": wl.name, "T": T, "d": d, "E": E, "k": k, "n": n,
                   "group": wl.group, "router_bias": wl.zipf > 0,
                   "l2": ("L2 flushed between steps (256 MB write), each step timed alone"
                          if flush is not None else
                          "inputs larger than L2 (3.4 GB of weights), no flush"),
                   "launch": "one CUDA graph per forward" if graph is not None else "eager",
                   "parallelism": f"replicas x{world}"},
        "layer_tflops": round(layer_flops / (ms_step / 1e3) / 1e12, 1),
        "step_ms": {"min": round(min(step_ms), 4), "median": round(statistics.median(step_ms), 4),
                    "max": round(max(step_ms), 4)},
        "stage_ms": {k_: round(v, 4) for k_, v in stage_ms.items()},
        "roofline": roof,
        "layer_roofline": layer_roof,
        "e2e": {"value": round(tokens / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 2},
        "gpu_launches": launches_per_step(T, d, E) * args.steps,
        "clocks": clk,
    }
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, inp, args.cpu_tokens)
    return out


# --------------------------------------------------------------------------- oracle
def cpu_baseline(wl, inp, ntok):
    import oracle
    ntok = min(ntok, wl.T)
    toks = np.random.default_rng(99).choice(wl.T, ntok, replace=False)
    oracle.lib()
    t0 = time.perf_counter()
    oracle.moe_forward(inp, wl.k, wl.group, tokens=toks)
    dt = time.perf_counter() - t0
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": round(ntok / dt, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{ntok} of {wl.T} tokens (seeded); the oracle's cost per token does "
                      f"not depend on T", "seconds": round(dt, 2)}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    import oracle
    inp = make_inputs(wl)
    oracle.lib()
    ntok = min(args.ref_tokens, wl.T)
    rng = np.random.default_rng(98)
    for _ in range(args.warmup):
        oracle.moe_forward(inp, wl.k, wl.group, tokens=rng.choice(wl.T, 2, replace=False))
    times = []
    for _ in range(args.steps):
        toks = rng.choice(wl.T, ntok, replace=False)
        t0 = time.perf_counter()
        oracle.moe_forward(inp, wl.k, wl.group, tokens=toks)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = ntok * args.steps / total
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    sample = f"{ntok} seeded tokens of the {wl.T}-token batch per step"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": wl.name, "T": wl.T, "d": wl.d, "E": wl.E, "k": wl.k,
                       "n": wl.n, "group": wl.group},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="large", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=256)
    ap.add_argument("--ref-tokens", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override T (profiling cases; not a bench line)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override E (profiling cases; not a bench line)")
    ap.add_argument("--only-forward", action="store_true",
                    help="time the forward only (fewer launches under a profiler)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    wl = WORKLOADS[args.workload]
    if args.tokens or args.experts:
        from moe_inputs import Workload
        wl = Workload(**{**wl.__dict__, "T": args.tokens or wl.T, "E": args.experts or wl.E,
                         "name": f"{wl.name}_T{args.tokens or wl.T}_E{args.experts or wl.E}"})
    if wl.chunk and wl.T > wl.chunk:
        # a chunked workload is timed one chunk (the largest) at a time
        from moe_inputs import Workload
        wl = Workload(**{**wl.__dict__, "T": wl.chunk, "name": wl.name + "_chunk"})
    res = run_reference(args, wl) if args.impl == "reference" else run_ours(args, wl)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
