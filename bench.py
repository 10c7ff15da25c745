#!/usr/bin/env python3
"""Benchmark of the MoE expert layer (route -> permute -> int4 grouped GEMMs
with SwiGLU -> combine) through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--sustain-s S] [--no-secondary]

One step = one strata_moe_forward over one batch of the workload (default:
the 6144-token prefill chunk, d=4096, 512 experts, top-10, n=1024, int4 with
group 64).  Inputs are seeded synthetic tensors resident in HBM; the weights
(3.4 GB) exceed the 126 MB L2, so no flush is needed between steps.  Prints one
JSON line.  With N > 1 (torchrun), every rank runs an independent replica
(the layer shards by token batches with no exchange); the time is the max over
ranks and `value` the total tokens of all ranks per second.

At N = 1 the line also carries
  * `secondary`: the other workloads of the same model family, each timed on
    its own inputs -- the 4-token verify batch and the 1-token decode step
    (HBM roofline over the weights they touch), the 512-token default batch
    (both rooflines) and the whole 34,000-token skewed prompt as six chunks
    (tokens/s = 34,000 / sum of chunk times, per-chunk expert load);
  * `sustained`: the headline forward run back to back for --sustain-s
    seconds (default 60) with the clocks sampled (NVML every 5 ms, else
    nvidia-smi every 200 ms): the rate, the median SM clock, time x clock,
    and step times binned by clock.

--impl reference times the fp64 CPU oracle on a bounded token sample of the
same workload on the host cores (rank 0 only).
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_inputs import (ATTN_WORKLOADS, WORKLOADS, Workload, chunk_sizes,  # noqa: E402
                        make_attention, make_inputs)

METRIC = "MoE-layer tokens/s at T=6144, 512 experts top-10; % of tensor/HBM roofline"
# Sources each profiled kernel is built from: its DRAM counters in
# profiles/traffic.json stand only while these files are unchanged.
KERNEL_SOURCES = {
    "gemm_gate_up_large": ["local_moe_route_b200/csrc/gemm_tc.cu",
                           "local_moe_route_b200/csrc/dequant.cuh",
                           "local_moe_route_b200/csrc/common.cuh"],
    "gemm_gate_up_verify4": ["local_moe_route_b200/csrc/gemm_decode.cu",
                             "local_moe_route_b200/csrc/common.cuh"],
}
WEIGHTS = ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples the SM clock, power and throttle reasons while a timed region
    runs: through NVML every 5 ms when it is available (a 100 ms timed
    region then has about 20 samples), else nvidia-smi every 200 ms.  Every
    sample is kept as an nvidia-smi CSV line (FIELDS order) with the host
    time it was taken."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    NVML_PERIOD_S = 0.005

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.nvml = None
        self.lines = []          # (host time, csv line)

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.nvml = (pynvml, handle)
            self.stop_event = threading.Event()
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    @classmethod
    def nvml_line(cls, nv, handle, index):
        """One sample from NVML in the CSV form nvidia-smi prints for FIELDS."""
        sm = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
        mx = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
        try:
            pw = "%.2f" % (nv.nvmlDeviceGetPowerUsage(handle) / 1000.0)
        except Exception:
            pw = "[N/A]"
        mask = nv.nvmlDeviceGetCurrentClocksEventReasons(handle)
        bits = (nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap)
        flags = ["Active" if mask & b else "Not Active" for b in bits]
        return ", ".join([str(index), str(sm), str(mx), pw, "0x%016x" % mask] + flags)

    def _poll(self):
        nv, handle = self.nvml
        while not self.stop_event.is_set():
            try:
                self.lines.append((time.time(), self.nvml_line(nv, handle, self.index)))
            except Exception:
                return
            time.sleep(self.NVML_PERIOD_S)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.nvml is not None:
            self.stop_event.set()
            self.thread.join(timeout=5)
            try:
                self.nvml[0].nvmlShutdown()
            except Exception:
                pass
            return self.summarise([ln for _, ln in self.lines])
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        return self.summarise([ln for _, ln in self.lines])

    @classmethod
    def parse(cls, line):
        """(sm MHz, max MHz, power W, set of active reasons) or None."""
        f = [x.strip() for x in line.split(",")]
        if len(f) < 9:
            return None
        try:
            sm, mx = float(f[1]), float(f[2])
        except ValueError:
            return None
        try:
            pw = float(f[3])
        except ValueError:
            pw = None
        reasons = {nm for nm, v in zip(cls.REASONS, f[5:9]) if v.lower() == "active"}
        return sm, mx, pw, reasons

    @classmethod
    def summarise(cls, lines):
        """Median SM clock under load, the maximum clock and the throttle
        reasons seen active, from nvidia-smi CSV lines in FIELDS order."""
        sm, mx, reasons = [], None, set()
        for line in lines:
            p = cls.parse(line)
            if p is None:
                continue
            sm.append(p[0])
            mx = p[1]
            reasons |= p[3]
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
    for n in WEIGHTS:
        L[n] = t(inp[n])
    return L


def fused_decode(T, d, E, k, n, group):
    """Whether strata_moe_forward runs the batch as one persistent launch
    (mirrors the library's rule for batches of at most four tokens)."""
    if not (1 <= T <= 4 and k <= 32 and E <= 1024 and E % 8 == 0 and group in (32, 64, 128)
            and d % 1024 == 0 and d <= 4096 and n % 256 == 0
            and (n // group) % 8 == 0 and n // group <= 64):
        return False
    xbytes = (T * (d + 8) * 2 + 1023) // 1024 * 1024
    smem = 3 * 16384 + xbytes + 8 * 32 * 8 * 4 + 128 + (2 * 128 + 4 * 1024 + 1 + 2 * 128 + 64) * 4
    return smem + 1024 <= 113 * 1024


def launches_per_step(T, d, E, k=10, n=1024, group=64):
    """Kernel launches of one strata_moe_forward (mirrors the dispatch rules)."""
    if fused_decode(T, d, E, k, n, group):
        return 1             # the whole layer in one kernel (plus a 16-byte memset)
    c = 2                    # router logits + top-k/softmax
    tc_router = T >= 128 and E % 128 == 0
    if not tc_router and T <= 16 and d // 32 > 1:
        c += 1               # sum of the K-split partial logits
    c += 3                   # permutation: histogram, scan, scatter
    c += 1                   # expert work lists
    c += 2 if T > 8 else 1   # gate/up (+ fp16 copy of x on the tensor-core path)
    c += 1                   # down
    c += 1                   # combine
    return c


def expert_bytes(wl):
    """Packed int4 codes and fp16 group scales of one expert's three matrices."""
    return 3 * wl.n * wl.d // 2 + 3 * wl.n * (wl.d // wl.group) * 2


def layer_flops(wl, T):
    """Algorithmic FLOPs of the layer for T tokens: the k chosen experts'
    three projections plus the router."""
    return 2.0 * T * wl.k * 3 * wl.d * wl.n + 2.0 * T * wl.d * wl.E


def layer_hbm_bytes(wl, T, touched):
    """Algorithmic bytes: weights of the touched experts, W_r, x and y."""
    return touched * expert_bytes(wl) + wl.d * wl.E * 2 + 2 * T * wl.d * 2


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


# --------------------------------------------------------------------------- timing
class LayerRun:
    """One workload resident on the device, called through strata_moe_forward.
    Batches of at most 64 tokens replay the forward as one CUDA graph (ten
    short kernels would otherwise wait on host launch overhead) and, since
    the weights they touch can stay in L2 from one step to the next, are
    timed one step at a time after a 256 MB write that evicts L2."""

    def __init__(self, sm, wl, inp, dev, T=None):
        import torch
        self.sm, self.wl, self.dev = sm, wl, dev
        self.T = wl.T if T is None else T
        self.L = device_layer(inp, dev)
        self.dims = wl.dims(self.T)
        self.ws = sm.workspace(self.dims, dev)
        self.y = torch.empty((self.T, wl.d), dtype=torch.bfloat16, device=dev)
        self.q4 = [(self.L[n + "_q"], self.L[n + "_s"]) for n in ("gate", "up", "down")]
        self.graph = None
        self.flush = None
        if self.T <= 64:
            self.forward()
            torch.cuda.synchronize()
            self.graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.graph):
                self.forward()
            torch.cuda.synchronize()
            self.flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)

    def forward(self, x=None, out=None, T=None, ids=None):
        import torch
        dims = self.dims if T is None else self.wl.dims(T)
        st = self.sm.strata_moe_forward(self.L["x"] if x is None else x, self.L["w_router"],
                                        self.L["bias"], *self.q4, dims,
                                        self.y if out is None else out, ids, None, self.ws,
                                        stream=torch.cuda.current_stream())
        if st != self.sm.STRATA_OK:
            raise self.sm.StrataError(st, "forward")

    def step(self):
        if self.graph is not None:
            self.graph.replay()
        else:
            self.forward()

    def time(self, steps):
        """Per-step device times (ms), CUDA events on the launching stream."""
        import torch
        stream = torch.cuda.current_stream()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * steps)]
        for i in range(steps):
            if self.flush is not None:
                self.flush.zero_()
            ev[2 * i].record(stream)
            self.step()
            ev[2 * i + 1].record(stream)
        torch.cuda.synchronize()
        return [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(steps)]

    def touched(self):
        """Experts the batch routes to (from one forward's ids)."""
        import torch
        ids = torch.empty((self.T, self.wl.k), dtype=torch.int32, device=self.dev)
        self.forward(ids=ids)
        torch.cuda.synchronize()
        return ids.cpu().numpy()


def expert_load(ids, E):
    counts = np.bincount(ids.ravel(), minlength=E)
    used = counts[counts > 0]
    return {"experts_touched": int(used.size), "rows_max": int(used.max()),
            "rows_mean_touched": round(float(used.mean()), 2),
            "rows_mean_all": round(float(counts.mean()), 2)}


def roof(achieved, peak, unit, bound, kind, **extra):
    out = {"bound": bound, "achieved": round(achieved, 1), "peak": peak, "unit": unit,
           "frac": round(achieved / peak, 4), "peak_kind": kind}
    out.update(extra)
    return out


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
    R = LayerRun(sm, wl, inp, dev)
    L, dims, ws, y = R.L, R.dims, R.ws, R.y
    T, d, k, n, E = wl.T, wl.d, wl.k, wl.n, wl.E
    S = T * k
    gate, up, down = R.q4
    stream = torch.cuda.current_stream()
    forward = R.forward

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- headline: K forwards, device time
    for _ in range(args.warmup):
        R.step()
    clocks = ClockSampler(dev.index) if rank == 0 else None
    barrier()
    if clocks:
        clocks.start()
        time.sleep(0.3)
    if R.flush is None:
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        ev0.record(stream)
        step_ev[0].record(stream)
        for i in range(args.steps):
            R.step()
            step_ev[i + 1].record(stream)
        ev1.record(stream)
        barrier()
        step_ms = [step_ev[i].elapsed_time(step_ev[i + 1]) for i in range(args.steps)]
        total_ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
    else:
        # the touched weights would stay in L2 from one step to the next:
        # overwrite L2 between steps and time each step alone
        step_ms = R.time(args.steps)
        barrier()
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
        if R.flush is not None:
            R.flush.zero_()
        staged(evs)
        torch.cuda.synchronize()
        for i, nm in enumerate(names):
            per[nm].append(evs[i].elapsed_time(evs[i + 1]))
    stage_ms = {nm: statistics.mean(v) for nm, v in per.items()}

    e2e_ms = max_over_ranks(time_e2e(R, inp, args, stream, barrier), dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    hbm, tf_burst, tf_sus, peak_kind = measured_peaks()
    tokens = T * args.steps * world
    value = job_throughput(T * args.steps, world, total_ms)
    ms_step = total_ms / args.steps
    ids_np = R.touched()
    touched = int(np.unique(ids_np).size)
    lflops = layer_flops(wl, T)
    lbytes = layer_hbm_bytes(wl, T, touched)
    if fused_decode(T, d, E, k, n, wl.group):
        # the forward is one kernel: its roofline is the layer's, over HBM
        roofline = roof(lbytes / (ms_step / 1e3) / 1e9, hbm, "GB/s", "hbm",
                        f"{peak_kind} copy bandwidth",
                        kernel="moe_decode_fused_kernel<G> (the whole layer, one launch)",
                        algorithmic_per_launch=lbytes, traffic=None)
    elif T > 8:
        # dominant kernel: gate/up grouped GEMM; algorithmic FLOPs per launch
        flops = 2.0 * S * 2 * d * n
        roofline = roof(flops / (stage_ms["gate_up"] / 1e3) / 1e12, tf_burst, "TFLOP/s", "tensor",
                        f"{peak_kind} bf16 dense burst (fp16 dense is the same rate)",
                        kernel="gate/up step: " + gate_up_kernels(T),
                        algorithmic_per_launch=flops,
                        traffic=profiled_traffic("gemm_gate_up_" + wl.name))
    else:
        # gate+up share of the touched experts' weight bytes
        bytes_ = touched * expert_bytes(wl) * 2 / 3
        roofline = roof(bytes_ / (stage_ms["gate_up"] / 1e3) / 1e9, hbm, "GB/s", "hbm",
                        f"{peak_kind} copy bandwidth",
                        kernel="gate/up step: " + gate_up_kernels(T),
                        algorithmic_per_launch=bytes_,
                        traffic=profiled_traffic("gemm_gate_up_" + wl.name))
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int4xfp16",
        "data": "synthetic (seeded, shapes of the pages' workload)",
        "config": {"workload": wl.name, "T": T, "d": d, "E": E, "k": k, "n": n,
                   "group": wl.group, "router_bias": wl.zipf > 0,
                   "l2": ("L2 flushed between steps (256 MB write), each step timed alone"
                          if R.flush is not None else
                          "inputs larger than L2 (3.4 GB of weights), no flush"),
                   "launch": "one CUDA graph per forward" if R.graph is not None else "eager",
                   "parallelism": f"replicas x{world}"},
        "layer_tflops": round(lflops / (ms_step / 1e3) / 1e12, 1),
        "step_ms": {"min": round(min(step_ms), 4), "median": round(statistics.median(step_ms), 4),
                    "max": round(max(step_ms), 4)},
        "stage_ms": {k_: round(v, 4) for k_, v in stage_ms.items()},
        "roofline": roofline,
        "layer_roofline": {
            "tensor": roof(lflops / (ms_step / 1e3) / 1e12, tf_burst, "TFLOP/s", "tensor",
                           f"{peak_kind} bf16 dense burst", flops_per_step=lflops),
            "hbm": roof(lbytes / (ms_step / 1e3) / 1e9, hbm, "GB/s", "hbm",
                        f"{peak_kind} copy bandwidth", bytes_per_step=lbytes,
                        experts_touched=touched)},
        "e2e": {"value": round(tokens / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 2},
        "gpu_launches": launches_per_step(T, d, E, k, n, wl.group) * args.steps,
        "clocks": clk,
    }
    if world == 1 and not args.no_secondary:
        out["secondary"] = {}
        for name in ("verify4", "decode1", "default", "skewed"):
            if name != wl.name:
                out["secondary"][name] = run_secondary(sm, dev, WORKLOADS[name], args)
        for name in ("attn_verify4", "attn_decode1"):
            out["secondary"][name] = run_secondary_attention(sm, dev, ATTN_WORKLOADS[name], args)
    if world == 1 and args.sustain_s > 0:
        out["sustained"] = run_sustained(R, args.sustain_s, dev, tf_burst, tf_sus, peak_kind)
    if not args.no_cpu_baseline:
        R.forward()
        out["cpu_baseline"] = cpu_baseline(wl, inp, args.cpu_tokens, R.y)
    return out


def gate_up_kernels(T):
    if T > 8:
        return ("work lists + grouped fp16 copy of x + moe_gemm_q4_tc_kernel<0,0,1> "
                "(gate/up + SwiGLU), one entry-point call")
    return "work lists + moe_gemm_q4_decode_kernel<2, G> (gate/up + SwiGLU), one entry-point call"


def time_e2e(R, inp, args, stream, barrier):
    """Same forward with the host -> device copy of x (pinned memory) and the
    device -> host copy of y inside the timed region, every step."""
    import torch
    T, d = R.T, R.wl.d
    x_host = torch.from_numpy(inp["x"]).view(torch.bfloat16).pin_memory()
    if R.flush is not None:
        # small batches: one step at a time, L2 flushed before each, each
        # step (copy in, forward, copy out) timed alone
        y_host = torch.empty((T, d), dtype=torch.bfloat16).pin_memory()
        x_dev = torch.empty_like(R.L["x"])
        for _ in range(args.warmup):
            x_dev.copy_(x_host, non_blocking=True)
            R.forward(x_dev)
            y_host.copy_(R.y, non_blocking=True)
        barrier()
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        for a_, b_ in pairs:
            R.flush.zero_()
            a_.record(stream)
            x_dev.copy_(x_host, non_blocking=True)
            R.forward(x_dev)
            y_host.copy_(R.y, non_blocking=True)
            b_.record(stream)
        barrier()
        return sum(a_.elapsed_time(b_) for a_, b_ in pairs)
    # large batches: copies pipelined against compute.  Step i's input is
    # copied in on one stream and its output copied out on another while
    # the forward of the neighbouring step runs; two device buffers each.
    y_host = [torch.empty((T, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(R.L["x"]) for _ in range(2)]
    y_dev = [torch.empty_like(R.y) for _ in range(2)]
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
        R.forward(x_dev[b_], out=y_dev[b_])
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
    return e0.elapsed_time(e1)


# --------------------------------------------------------------------------- secondary
def run_secondary(sm, dev, wl, args):
    """One other workload on its own seeded inputs: tokens/s and the layer's
    rooflines.  The skewed prompt runs as its chunks, one forward each."""
    import gc
    import torch
    hbm, tf_burst, _, peak_kind = measured_peaks()
    inp = make_inputs(wl)
    sizes = chunk_sizes(wl.T, wl.chunk)
    R = LayerRun(sm, wl, inp, dev, T=max(sizes))
    res = {"T": wl.T, "d": wl.d, "E": wl.E, "k": wl.k, "n": wl.n, "group": wl.group}
    steps = args.secondary_steps
    if len(sizes) == 1:
        for _ in range(args.warmup):
            R.step()
        ms = R.time(steps)
        med = statistics.median(ms)
        ids = R.touched()
        load = expert_load(ids, wl.E)
        lflops = layer_flops(wl, wl.T)
        lbytes = layer_hbm_bytes(wl, wl.T, load["experts_touched"])
        res.update({
            "tokens_per_s": round(wl.T / (med / 1e3), 1), "ms_per_step": round(med, 4),
            "steps": steps,
            "step_ms": {"min": round(min(ms), 4), "max": round(max(ms), 4)},
            "launch": "one CUDA graph per forward" if R.graph is not None else "eager",
            "l2": "flushed (256 MB write) before each step" if R.flush is not None else
                  "weights larger than L2, no flush",
            "layer_roofline": {
                "hbm": roof(lbytes / (med / 1e3) / 1e9, hbm, "GB/s", "hbm",
                            f"{peak_kind} copy bandwidth", bytes_per_step=lbytes),
                "tensor": roof(lflops / (med / 1e3) / 1e12, tf_burst, "TFLOP/s", "tensor",
                               f"{peak_kind} bf16 dense burst", flops_per_step=lflops)},
            "expert_load": load,
        })
    else:
        # the whole prompt, chunk by chunk; per repetition the chunk times add
        starts = np.concatenate([[0], np.cumsum(sizes)[:-1]]).astype(int)
        xs = [R.L["x"][s0:s0 + m] for s0, m in zip(starts, sizes)]
        ys = [torch.empty((m, wl.d), dtype=torch.bfloat16, device=dev) for m in sizes]
        stream = torch.cuda.current_stream()

        def prompt(evs=None):
            for c, m in enumerate(sizes):
                if evs is not None:
                    evs[c].record(stream)
                R.forward(xs[c], out=ys[c], T=m)
            if evs is not None:
                evs[len(sizes)].record(stream)

        for _ in range(max(1, args.warmup // 2)):
            prompt()
        reps = max(3, steps // 10)
        per_chunk = [[] for _ in sizes]
        totals = []
        for _ in range(reps):
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(sizes) + 1)]
            prompt(evs)
            torch.cuda.synchronize()
            t = [evs[c].elapsed_time(evs[c + 1]) for c in range(len(sizes))]
            for c in range(len(sizes)):
                per_chunk[c].append(t[c])
            totals.append(sum(t))
        med = statistics.median(totals)
        chunks = []
        for c, m in enumerate(sizes):
            ids = torch.empty((m, wl.k), dtype=torch.int32, device=dev)
            R.forward(xs[c], out=ys[c], T=m, ids=ids)
            torch.cuda.synchronize()
            load = expert_load(ids.cpu().numpy(), wl.E)
            load.update({"T": m, "ms": round(statistics.median(per_chunk[c]), 4)})
            chunks.append(load)
        lflops = layer_flops(wl, wl.T)
        res.update({
            "tokens_per_s": round(wl.T / (med / 1e3), 1),
            "ms_per_prompt": round(med, 4), "repetitions": reps,
            "chunks": chunks, "launch": "eager, one forward per chunk",
            "layer_roofline": {
                "tensor": roof(lflops / (med / 1e3) / 1e12, tf_burst, "TFLOP/s", "tensor",
                               f"{peak_kind} bf16 dense burst", flops_per_prompt=lflops)},
        })
    assert sm.strata_moe_device_status() == sm.STRATA_OK
    del R
    gc.collect()
    torch.cuda.empty_cache()
    return res


def run_secondary_attention(sm, dev, aw, args):
    """Attention over the indexer-selected KV rows of a 34,000-token cache:
    device time of strata_sparse_attention (two kernels), L2 overwritten
    before every call, HBM roofline over the selected K and V rows."""
    import torch
    hbm, _, _, peak_kind = measured_peaks()
    a = make_attention(aw.T, aw.L, aw.Hq, aw.Hkv, aw.D, aw.P, aw.seed)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    q, k, v, idx = t(a["q"]), t(a["k"]), t(a["v"]), t(a["idx"])
    dims = dict(T=aw.T, L=aw.L, Hq=aw.Hq, Hkv=aw.Hkv, D=aw.D, P=aw.P)
    out = torch.empty((aw.T, aw.Hq, aw.D), dtype=torch.bfloat16, device=dev)
    ws = sm.attention_workspace(dims, dev)
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def call():
        sm.check(sm.strata_sparse_attention(q, k, v, idx, dims, 0.0, out, ws,
                                            stream=torch.cuda.current_stream()))

    for _ in range(args.warmup):
        call()
    # one call captured as a CUDA graph: the events then bracket the two
    # kernels alone, not the host's time to marshal and launch them
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        graph.replay()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.secondary_steps)]
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    assert sm.strata_moe_device_status() == sm.STRATA_OK
    ms = [e0.elapsed_time(e1) for e0, e1 in ev]
    med = statistics.median(ms)
    valid = int(np.sum(a["idx"] >= 0))
    rows_bytes = valid * aw.Hkv * aw.D * 2 * 2            # selected K and V rows
    bytes_ = rows_bytes + a["idx"].nbytes + 2 * aw.T * aw.Hq * aw.D * 2
    return {"T": aw.T, "L": aw.L, "Hq": aw.Hq, "Hkv": aw.Hkv, "D": aw.D, "P": aw.P,
            "ms_per_call": round(med, 5), "steps": len(ms),
            "queries_per_s": round(aw.T / (med / 1e3), 1),
            "l2": "flushed (256 MB write) before each call",
            "launch": "one CUDA graph per call",
            "roofline": roof(bytes_ / (med / 1e3) / 1e9, hbm, "GB/s", "hbm",
                             f"{peak_kind} copy bandwidth", bytes_per_call=bytes_,
                             kernel="sparse_attn_split_kernel + sparse_attn_combine_kernel"),
            "dense_cache_bytes": 2 * aw.L * aw.Hkv * aw.D * 2}


# --------------------------------------------------------------------------- sustained
def run_sustained(R, seconds, dev, tf_burst, tf_sus, peak_kind):
    """The headline forward back to back for `seconds`, clocks sampled as in
    ClockSampler.  Events every `block` steps give the step time over the run;
    each clock sample is paired with the block running when it was taken."""
    import torch
    stream = torch.cuda.current_stream()
    block = 20 if R.T > 64 else 200
    clocks = ClockSampler(dev.index)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    t_host0 = time.time()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    evs = []
    while time.time() - t_host0 < seconds:
        for _ in range(block):
            R.step()
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        evs.append(e)
        if len(evs) > 4:
            evs[-4].synchronize()      # keep the host at most a few blocks ahead
    torch.cuda.synchronize()
    clocks.stop()
    ends = [ev0.elapsed_time(e) for e in evs]            # ms since start, per block
    nsteps = block * len(evs)
    total = ends[-1]
    starts = [0.0] + ends[:-1]
    block_ms = [(b - a) / block for a, b in zip(starts, ends)]
    samples = []
    for ts, line in clocks.lines:
        p = ClockSampler.parse(line)
        t = (ts - t_host0) * 1e3
        if p is None or t < 0 or t > total:
            continue
        i = int(np.searchsorted(ends, t))
        samples.append((p[0], block_ms[min(i, len(block_ms) - 1)], p[2], p[3]))
    summ = ClockSampler.summarise([ln for _, ln in clocks.lines]) or {}
    bins = {}
    for mhz, ms, _, _ in samples:
        key = int(mhz // 100 * 100)
        bins.setdefault(key, []).append(ms)
    flops = layer_flops(R.wl, R.T)
    ms_step = total / nsteps
    med_mhz = summ.get("sm_mhz")
    watts = [s[2] for s in samples if s[2] is not None]
    return {
        "seconds": round(total / 1e3, 1), "steps": nsteps, "ms_per_step": round(ms_step, 4),
        "tokens_per_s": round(R.T * nsteps / (total / 1e3), 1),
        "layer_tflops": round(flops / (ms_step / 1e3) / 1e12, 1),
        "frac_of_burst": round(flops / (ms_step / 1e3) / 1e12 / tf_burst, 4),
        "frac_of_sustained": (round(flops / (ms_step / 1e3) / 1e12 / tf_sus, 4)
                              if tf_sus else None),
        "peak_kind": peak_kind,
        "first_10pct_ms_per_step": round(statistics.mean(block_ms[:max(1, len(block_ms) // 10)]), 4),
        "last_10pct_ms_per_step": round(statistics.mean(block_ms[-max(1, len(block_ms) // 10):]), 4),
        "clocks": summ,
        "ms_per_step_x_median_mhz": round(ms_step * med_mhz, 1) if med_mhz else None,
        "power_w_median": round(statistics.median(watts), 1) if watts else None,
        "by_clock_mhz": {str(k_): {"samples": len(v), "ms_per_step": round(statistics.mean(v), 4)}
                         for k_, v in sorted(bins.items())},
    }


# --------------------------------------------------------------------------- oracle
def cpu_baseline(wl, inp, ntok, y_dev=None):
    """The fp64 oracle on a seeded token sample, on all host cores.  With the
    GPU's output y_dev of the same batch, the sample also gives the parity
    of those tokens: the gate (error beyond one bf16 rounding), the literal
    max-abs error and the distance from the correctly rounded oracle."""
    import oracle
    ntok = min(ntok, wl.T)
    toks = np.sort(np.random.default_rng(99).choice(wl.T, ntok, replace=False))
    oracle.lib()
    t0 = time.perf_counter()
    ref = oracle.moe_forward(inp, wl.k, wl.group, tokens=toks)
    dt = time.perf_counter() - t0
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    out = {"value": round(ntok / dt, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
           "sample": f"{ntok} of {wl.T} tokens (seeded); the oracle's cost per token does "
                     f"not depend on T", "seconds": round(dt, 2)}
    if y_dev is not None:
        import torch
        bits = y_dev.view(torch.int16).cpu().numpy().view(np.uint16)[toks]
        got = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        y = ref["y"]
        r = float(np.sqrt(np.mean(y * y)))
        m, e = np.frexp(y)
        rounded = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)      # RNE to bf16
        half_ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(y), 1e-300))) - 8)
        out["parity_of_sample"] = {
            "gate": round(float(np.max(np.abs(got - y) - half_ulp) / r), 5),
            "raw_max_abs": round(float(np.max(np.abs(got - y)) / r), 5),
            "exactly_rounded_raw_max_abs": round(float(np.max(np.abs(rounded - y)) / r), 5),
            "vs_rounded_oracle_max_abs": round(float(np.max(np.abs(got - rounded)) / r), 5),
            "limit": 1.5e-2, "unit": "RMS of the oracle output"}
    return out


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
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the other workloads (N = 1 only)")
    ap.add_argument("--secondary-steps", type=int, default=50)
    ap.add_argument("--sustain-s", type=float, default=60.0,
                    help="seconds of back-to-back forwards after the timed steps (N = 1; 0: off)")
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
        wl = Workload(**{**wl.__dict__, "T": args.tokens or wl.T, "E": args.experts or wl.E,
                         "name": f"{wl.name}_T{args.tokens or wl.T}_E{args.experts or wl.E}"})
        args.no_secondary = True
        args.sustain_s = 0
    if wl.chunk and wl.T > wl.chunk:
        # a chunked workload's headline is one chunk (the largest); the whole
        # prompt is timed among the secondary results
        wl = Workload(**{**wl.__dict__, "T": wl.chunk, "name": wl.name + "_chunk"})
    res = run_reference(args, wl) if args.impl == "reference" else run_ours(args, wl)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
