#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 linear layer on B200; prints ONE JSON line.

Step = forward + backward of all seven QLoRA linears of one Llama-65B-shaped
decoder layer (q, k, v, o 8192x8192; gate, up 8192->22016; down 22016->8192;
all NF4 with double quantization, LoRA r = 64, alpha = 16 on every one),
M = 2048 tokens, each projection on its own seeded input: per projection the
hot path's kernels (LoRA down-projection, fused dequant GEMM forward, du,
fused dequant GEMM dx, dA and dB).  The frozen weights are quantized before
timing; quantizing all seven is timed separately and reported in the same
line.  Components (7B attention and MLP fwd+bwd, the 70B few-token GEMV, the
quantizer variants, the adapter merge, LoRA dropout) follow on N = 1.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1: launched with torch.distributed.run, one rank per GPU; every rank runs
its own batch (data parallel, weak scaling) and the adapter gradients of the
layer (one flat fp32 buffer) are summed across ranks with one NCCL all-reduce
per step.  Time = max over ranks of the CUDA-event time of exactly K steps,
bracketed by barrier + synchronize.  `--impl reference` times the fp64 CPU
oracle (rank 0 only) on a bounded token sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_nf4_quantized_11_b200 import dp, synth, workloads  # noqa: E402

METRIC = "QLoRA linear fwd+bwd TFLOP/s and NF4 quant/GEMV GB/s, % of B200 roofline"
L2_BYTES = 126 * 2 ** 20
WL = workloads.LAYER_65B          # the largest configuration that fits one GPU
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------- helpers
def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-components", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only", choices=["quantize", "gemv", "workloads", "merge", "dropout", "layer_step",
                                       "q_proj_steps", "dropout_steps"],
                    default=None,
                    help="run one component measurement alone and print it (for profiling)")
    return ap.parse_args()


NOMINAL_BF16_TFLOPS = 2250.0      # dense bf16 tensor peak of one B200 (spec figure, for context)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# sources of the fused dequant GEMM kernels (the dominant kernel of the step)
GEMM_SOURCES = ("common.cuh", "gemm_pair_sm100.cuh", "gemm_sm100.cuh")


def source_hash(names=GEMM_SOURCES):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_nf4_quantized_11_b200", "csrc")
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources; otherwise None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        if t.get("source_hash") != source_hash():
            return None
        return t["kernels"][workload][kernel]["dram_bytes_per_launch"]
    except Exception:
        return None


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thr is not None:
            self._thr.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


# ---------------------------------------------------------------------------- our arm
def gemm_flops(kernel, M, n_in, n_out, r):
    """Algorithmic FLOPs of one launch of a fused dequant GEMM: the forward
    contracts [x | us] with [W0 | B] (K = in + r), dx [dh | du] with [W0 ; A]."""
    return 2.0 * M * (n_out * (n_in + r) if kernel == "gemm_fwd" else n_in * (n_out + r))


class LayerState:
    """One rank's device-resident copy of the headline workload: every
    projection's fp32 weight (for the quantizer figure), its NF4 weight, its
    own inputs x, dh, the adapters A, B, the outputs and the workspaces; the
    adapter gradients of all projections live in one flat buffer."""

    def __init__(self, q, wl, seed0, dev):
        self.q, self.wl, self.M, self.r, self.alpha = q, wl, wl.M[0], wl.r, wl.alpha
        self.shapes = [(n_in, n_out) for _, n_in, n_out in wl.projections]
        self.flat, grads = dp.layer_grad_buffers(self.r, self.shapes, dev)
        self.proj = []
        for i, ((label, n_in, n_out), (dA, dB)) in enumerate(zip(wl.projections, grads)):
            p = synth.problem(self.M, n_in, n_out, self.r, wl.w_std, wl.w_dist, seed=seed0 + i)
            c = {k: p[k].to(dev) for k in ("W", "x", "A", "B", "dh")}
            del p
            c["label"], c["n_in"], c["n_out"] = label, n_in, n_out
            c["w"] = q.alloc_nf4(n_out, n_in, dev)
            c["h"] = torch.empty(self.M, n_out, dtype=torch.bfloat16, device=dev)
            c["us"] = torch.empty(self.M, self.r, dtype=torch.bfloat16, device=dev)
            c["dx"] = torch.empty(self.M, n_in, dtype=torch.bfloat16, device=dev)
            c["dA"], c["dB"] = dA, dB
            self.proj.append(c)
        ws = lambda op: max(max(1, q.workspace_size(op, self.M, n_in, n_out, self.r))  # noqa: E731
                            for n_in, n_out in self.shapes)
        self.ws_f = torch.empty(ws(q.OP_LINEAR_FWD), dtype=torch.uint8, device=dev)
        self.ws_b = torch.empty(ws(q.OP_LINEAR_BWD), dtype=torch.uint8, device=dev)
        self.problems = self.make_problems(self.proj, [(c["dA"], c["dB"]) for c in self.proj])
        self.ws_gf, self.ws_gb = self.group_workspaces(self.problems, dev)
        self.ws_q = torch.empty(max(q.workspace_size(q.OP_QUANTIZE, 0, n_in, n_out, 0) for n_in, n_out in self.shapes),
                                dtype=torch.uint8, device=dev)
        self.quantize()
        torch.cuda.synchronize()

    def quantize(self):
        for c in self.proj:
            self.q.quantize_nf4(c["W"], out=c["w"], workspace=self.ws_q)

    def make_problems(self, bufs, grads):
        """One grouped-call problem per projection over the given x, dh, h,
        us, dx buffers and (dA, dB) gradient views."""
        return [self.q.LinearProblem(x=b["x"], w=c["w"], A=c["A"], B=c["B"], alpha=self.alpha, h=b["h"], us=b["us"],
                                     dh=b["dh"], dx=b["dx"], dA=dA, dB=dB)
                for c, b, (dA, dB) in zip(self.proj, bufs, grads)]

    def group_workspaces(self, problems, dev):
        q = self.q
        return tuple(torch.empty(max(1, q.linear_group_workspace_size(bwd, problems)), dtype=torch.uint8, device=dev)
                     for bwd in (False, True))

    def step(self, world=1, grouped=True, problems=None):
        """Forward and backward of every projection.  Grouped (the default):
        two grouped calls, whose rank-r kernels run beside the GEMMs;
        otherwise one linear_fwd + linear_bwd call per projection."""
        q, a = self.q, self.alpha
        if grouped:
            probs = self.problems if problems is None else problems
            q.linear_fwd_group(probs, workspace=self.ws_gf)
            q.linear_bwd_group(probs, workspace=self.ws_gb)
        else:
            for c in self.proj:
                q.linear_fwd(c["x"], c["w"], c["A"], c["B"], a, h=c["h"], us=c["us"], workspace=self.ws_f)
                q.linear_bwd(c["dh"], c["x"], c["us"], c["w"], c["A"], c["B"], a, dx=c["dx"], dA=c["dA"],
                             dB=c["dB"], workspace=self.ws_b)
        if world > 1:                       # data-parallel adapter-gradient sum, one all-reduce per layer
            dp.allreduce_adapter_grads(self.flat)

    def flops(self):
        return sum(workloads.fwd_bwd_flops(self.M, n_in, n_out, self.r) for n_in, n_out in self.shapes)

    def gemm_flops(self, kernel):
        return sum(gemm_flops(kernel, self.M, n_in, n_out, self.r) for n_in, n_out in self.shapes)

    def input_bytes(self):
        return sum(c[k].numel() * c[k].element_size() for c in self.proj for k in ("x", "dh")) + \
            sum(c["w"].nbytes() for c in self.proj)


def run_ours(args, world, rank, local):
    import bit_nf4_quantized_11_b200 as q
    q.load()
    dev = torch.device("cuda", local)
    L = LayerState(q, WL, 1000 * rank, dev)

    for _ in range(args.warmup):
        L.step(world)
    torch.cuda.synchronize()
    if q.last_device_status() != 0:
        raise RuntimeError("device wait timed out during warm-up")

    stream = torch.cuda.current_stream()

    def timed_region(per_kernel: bool, body, n):
        """n calls of body between barrier+synchronize, CUDA events on this
        stream; with per_kernel, the library also brackets each of its
        launches with events (the headline value comes from the region
        without them)."""
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        q.timing_reset()
        q.timing_enable(per_kernel)
        barrier(world)
        torch.cuda.synchronize()
        with ClockSampler(local) as clk:
            e0.record(stream)
            for _ in range(n):
                body()
            e1.record(stream)
            torch.cuda.synchronize()
        barrier(world)
        q.timing_enable(False)
        if q.last_device_status() != 0:
            raise RuntimeError("device wait timed out in the timed region")
        return max_over_ranks(e0.elapsed_time(e1), world), clk

    step = lambda: L.step(world)  # noqa: E731
    ms_max, clk = timed_region(False, step, args.steps)
    flops = L.flops()
    value = world * args.steps * flops / (ms_max * 1e-3) / 1e12

    # identical second region with per-kernel events: breakdown, launch count, roofline
    ms_events, _ = timed_region(True, step, args.steps)
    kern = {}
    launches = 0
    for name in q.KERNEL_NAMES:
        t, n = q.timing_collect(name)
        if n:
            kern[name] = {"ms_per_step": t / args.steps, "launches": n, "avg_us": 1e3 * t / n}
            launches += n
    total_k = sum(v["ms_per_step"] for v in kern.values())
    for v in kern.values():
        v["share"] = v["ms_per_step"] / total_k if total_k else None

    peaks, peak_src = load_peaks()
    dom = max(("gemm_fwd", "gemm_dx"), key=lambda k: kern.get(k, {}).get("ms_per_step", 0.0))
    launches_per_step = kern[dom]["launches"] / args.steps
    dom_flops = L.gemm_flops(dom) / launches_per_step            # mean algorithmic FLOPs per launch
    achieved = dom_flops / (kern[dom]["avg_us"] * 1e-6) / 1e12
    region_s = ms_max * 1e-3
    long_region = region_s >= 2.0
    peak = peaks["bf16_tflops_sustained"] if long_region else peaks["bf16_tflops"]
    roofline = {"kernel": dom, "bound": "tensor", "achieved": achieved,
                "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_source": ("bf16_tflops_sustained" if long_region else "bf16_tflops (burst)")
                               + f" of {peak_src}: the timed region lasts {region_s:.2f} s "
                               + ("(seconds-long, power-capped)" if long_region else "(well under the seconds-long "
                                  "loop the sustained figure was measured on)"),
                "timing": "mean CUDA-event duration of the kernel's launches (one per projection and step) in a "
                          "second K-step region identical to the timed one, events recorded on the launching "
                          "stream; achieved = mean algorithmic FLOPs per launch / mean duration",
                "frac_of_burst_peak": achieved / peaks["bf16_tflops"],
                "frac_of_sustained_peak": achieved / peaks["bf16_tflops_sustained"],
                "frac_of_nominal": achieved / NOMINAL_BF16_TFLOPS,
                "flops_per_launch": dom_flops,
                "step_frac_of_peak": value / world / peak,
                "traffic": profiled_traffic(dom, WL.name)}

    # the same step as single calls per projection (no overlap of the rank-r
    # kernels with the GEMMs), for comparison
    ms_seq, clk_seq = timed_region(False, lambda: L.step(world, grouped=False), args.steps)
    sequential = {"what": "the same step as one linear_fwd + linear_bwd call per projection on one stream",
                  "ms_per_step": ms_seq / args.steps,
                  "TFLOP/s": world * args.steps * flops / (ms_seq * 1e-3) / 1e12,
                  "clocks": clk_seq.summary()}

    # quantizing all seven weights, timed on its own (3.24 GB of fp32 weights > L2)
    n_q = max(3, min(20, args.steps))
    ms_q, _ = timed_region(False, L.quantize, n_q)
    qbytes = sum(workloads.quant_bytes(n_out, n_in) for n_in, n_out in L.shapes)
    qgbs = world * n_q * qbytes / (ms_q * 1e-3) / 1e9
    quant = {"what": "NF4 + double quantization of the layer's seven fp32 weights "
                     f"({sum(a * b for a, b in L.shapes) / 1e6:.1f} M weights)",
             "ms": ms_q / n_q, "GB/s": qgbs, "unit": "GB/s", "bytes": qbytes,
             "bound": "hbm", "peak": peaks["hbm_gbs"], "frac": qgbs / world / peaks["hbm_gbs"],
             "peak_source": f"hbm_gbs of {peak_src}",
             "bytes_rule": "4 B read + 0.5 B codes + 1/64 B scale codes + 4 B per 256 blocks per weight"}

    e2e = None if args.no_e2e else measure_e2e(q, args, L, world, dev)

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": f"synthetic: seeded N(0,1) bf16 activations and output grads per projection, N(0,{WL.w_std}^2) fp32 "
                "weights quantized to NF4 + double quant, U(+-1/sqrt(in)) A, N(0,0.01^2) B",
        "config": {"workload": WL.name,
                   "projections": [f"{lab} {a}->{b}" for lab, a, b in WL.projections],
                   "tokens_per_gpu": L.M, "r": L.r, "alpha": L.alpha, "global_tokens": L.M * world,
                   "parallelism": f"dp{world}",
                   "l2": f"inputs larger than L2: one step reads {L.input_bytes() / 2**20:.0f} MiB of distinct "
                         "weights and activations (> 126 MiB L2), no projection's data is reused within a step",
                   "flops_per_step_per_gpu": flops},
        "roofline": roofline,
        "quantize": quant,
        "e2e": e2e,
        "gpu_launches": launches,
        "ms_per_step_with_kernel_events": ms_events / args.steps,
        "single_calls": sequential,
        "clocks": clk.summary(),
        "kernels": kern,
    }
    del L
    torch.cuda.empty_cache()
    return line


def measure_e2e(q, args, L, world, dev):
    """Same step through the public API with inputs in pinned host memory:
    every step copies each projection's x, dh host->device and its h, dx
    device->host, and the layer's flat adapter gradients (dA, dB of all
    projections) device->host.  Projections are pipelined over two buffer
    sets on three streams (host->device copies, the layer, device->host
    copies), so the copies of one projection overlap the compute of its
    neighbours; every step's own copies are inside the timed region."""
    P = len(L.proj)
    n = max(3, min(10, args.steps // 5))
    bufs = []
    for c in L.proj:
        sets = []
        for _ in range(2):
            sets.append({"xh": c["x"].cpu().pin_memory(), "dhh": c["dh"].cpu().pin_memory(),
                         "x": torch.empty_like(c["x"]), "dh": torch.empty_like(c["dh"]),
                         "h": torch.empty_like(c["h"]), "us": torch.empty_like(c["us"]),
                         "dx": torch.empty_like(c["dx"]),
                         "h_host": torch.empty(c["h"].shape, dtype=torch.bfloat16).pin_memory(),
                         "dx_host": torch.empty(c["dx"].shape, dtype=torch.bfloat16).pin_memory()})
        bufs.append(sets)
    grads = [dp.layer_grad_buffers(L.r, L.shapes, dev) for _ in range(2)]
    g_host = [torch.empty(grads[0][0].numel(), dtype=torch.float32).pin_memory() for _ in range(2)]
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    loaded = [[ev(), ev()] for _ in range(P)]
    used = [[ev(), ev()] for _ in range(P)]
    computed = [[ev(), ev()] for _ in range(P)]
    drained = [[ev(), ev()] for _ in range(P)]
    g_done, g_drained = [ev(), ev()], [ev(), ev()]

    def step(i):
        k = i % 2
        flat, views = grads[k]
        for p, c in enumerate(L.proj):
            b = bufs[p][k]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(used[p][k])             # step i-2 no longer reads this input set
                b["x"].copy_(b["xh"], non_blocking=True)
                b["dh"].copy_(b["dhh"], non_blocking=True)
                loaded[p][k].record(s_in)
            with torch.cuda.stream(s_run):
                s_run.wait_event(loaded[p][k])
                if i >= 2:
                    s_run.wait_event(drained[p][k])         # step i-2's outputs are on the host
                    if p == 0:
                        s_run.wait_event(g_drained[k])      # and its gradients
                dA, dB = views[p]
                q.linear_fwd(b["x"], c["w"], c["A"], c["B"], L.alpha, h=b["h"], us=b["us"], workspace=L.ws_f)
                q.linear_bwd(b["dh"], b["x"], b["us"], c["w"], c["A"], c["B"], L.alpha, dx=b["dx"], dA=dA, dB=dB,
                             workspace=L.ws_b)
                used[p][k].record(s_run)
                computed[p][k].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[p][k])
                b["h_host"].copy_(b["h"], non_blocking=True)
                b["dx_host"].copy_(b["dx"], non_blocking=True)
                drained[p][k].record(s_out)
        with torch.cuda.stream(s_run):
            if world > 1:
                dp.allreduce_adapter_grads(flat)
            g_done[k].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(g_done[k])
            g_host[k].copy_(flat, non_blocking=True)
            g_drained[k].record(s_out)

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(n):
        step(i)
    s_in.wait_stream(s_out)
    e1.record(s_in)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    h2d = sum(c["x"].numel() * 2 + c["dh"].numel() * 2 for c in L.proj)
    d2h = sum(c["h"].numel() * 2 + c["dx"].numel() * 2 for c in L.proj) + 4 * grads[0][0].numel()
    return {"value": world * n * L.flops() / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n, "ms_per_step": ms / n,
            "pipeline": "per projection: 2 buffer sets on 3 streams, the host<->device copies of neighbouring "
                        "projections overlap the compute; the step ends when its last copy to the host is done"}


# ---------------------------------------------------------------------------- oracle legs
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


class OracleLayer:
    """The fp64 oracle set up once on one projection of the headline layer
    (its weight quantized and dequantized by the oracle itself).  The oracle
    is timed on a token sample through this projection: quantizing all seven
    of the layer's weights in fp64 NumPy would take minutes and ~10 GB of host
    memory, and the oracle's FLOP rate does not depend on which projection
    it runs."""

    PROJ = 0          # q_proj, 8192 x 8192

    def __init__(self, seed=0):
        from oracle import linear, nf4
        label, n_in, n_out = WL.projections[self.PROJ]
        self.label, self.linear, self.n_in, self.n_out, self.r, self.alpha = label, linear, n_in, n_out, WL.r, WL.alpha
        p = synth.problem(WL.M[0], n_in, n_out, WL.r, WL.w_std, WL.w_dist, seed + self.PROJ)
        qo = nf4.quantize(p["W"].numpy())
        self.Wd = nf4.dequantize(qo["codes"], qo["q8"], qo["step2"], qo["mean"])
        self.x = p["x"].float().numpy().astype("float64")
        self.dh = p["dh"].float().numpy().astype("float64")
        self.A = p["A"].float().numpy().astype("float64")
        self.B = p["B"].float().numpy().astype("float64")

    def step(self, m0, m):
        sl = slice(m0 % WL.M[0], m0 % WL.M[0] + m)
        x, dh = self.x[sl], self.dh[sl]
        self.linear.linear_fwd(x, self.Wd, self.A, self.B, self.alpha)
        self.linear.linear_bwd(dh, x, self.Wd, self.A, self.B, self.alpha)
        return workloads.fwd_bwd_flops(x.shape[0], self.n_in, self.n_out, self.r)

    def describe(self, m):
        return (f"fp64 NumPy oracle fwd+bwd of {m} of the {WL.M[0]} tokens through the layer's {self.label} "
                f"({self.n_out}x{self.n_in}, r={self.r}), the oracle's own NF4 weight")


def cpu_baseline(budget_s=15.0):
    ol = OracleLayer()
    t0 = time.perf_counter()
    ol.step(0, 32)
    per_tok = (time.perf_counter() - t0) / 32
    m = int(max(32, min(WL.M[0], budget_s / max(per_tok, 1e-9))))
    # whole samples repeated until about budget_s of work (one when it alone is longer)
    reps = max(1, int(budget_s / max(per_tok * m, 1e-9)))
    t0 = time.perf_counter()
    flops = sum(ol.step(0, m) for _ in range(reps))
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{ol.describe(m)}, {reps} time(s); {dt:.1f} s"}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    ol = OracleLayer()
    t0 = time.perf_counter()
    ol.step(0, 16)
    per_tok = (time.perf_counter() - t0) / 16
    budget = 120.0
    m = int(max(1, min(WL.M[0], budget / max(per_tok, 1e-9) / max(1, args.steps + args.warmup))))
    for i in range(args.warmup):
        ol.step(i * m, m)
    t0 = time.perf_counter()
    flops = 0.0
    for i in range(args.steps):
        flops += ol.step((args.warmup + i) * m, m)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    cores = blas_threads()
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same seeded inputs as the GPU arm)",
        "config": {"workload": WL.name, "sampled_projection": f"{ol.label} {ol.n_in}->{ol.n_out}",
                   "tokens_per_step": m, "r": ol.r, "alpha": ol.alpha},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{ol.describe(m)} per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------- components
def comp_quantize(q, dev, peaks, src, reps=3):
    """Quantizer and dequantizer on the 65B decoder layer's seven weights (3.2 GB fp32 > L2)."""
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    out = {}
    weights = []
    for i, (label, n_in, n_out) in enumerate(workloads.LAYER_65B.projections):
        W = synth.weight(n_out, n_in, workloads.LAYER_65B.w_std, seed=i).to(dev)
        weights.append((label, W, q.alloc_nf4(n_out, n_in, dev)))
    ws = torch.empty(max(q.workspace_size(q.OP_QUANTIZE, 0, W.shape[1], W.shape[0], 0)
                         for _, W, _ in weights), dtype=torch.uint8, device=dev)
    for _ in range(2):
        for _, W, w in weights:
            q.quantize_nf4(W, out=w, workspace=ws)
    torch.cuda.synchronize()
    a, b = ev(), ev()

    def region(per_kernel):
        q.timing_reset()
        q.timing_enable(per_kernel)
        a.record()
        for _ in range(reps):
            for _, W, w in weights:
                q.quantize_nf4(W, out=w, workspace=ws)
        b.record()
        torch.cuda.synchronize()
        q.timing_enable(False)
        return a.elapsed_time(b) / reps

    tot = region(False)                       # clean: no per-kernel events
    region(True)                              # same work, per-kernel split
    qbytes = sum(workloads.quant_bytes(*W.shape) for _, W, _ in weights)
    split = {}
    for name in ("quantize_blocks", "scale_mean_tree", "dq_scales"):
        t, n = q.timing_collect(name)
        split[name + "_ms"] = t / reps if n else None
    out["quantize_65b_layer"] = {
        "weights": sum(W.numel() for _, W, _ in weights), "ms": tot, "GB/s": qbytes / (tot * 1e-3) / 1e9,
        "frac_hbm": qbytes / (tot * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "kernels_with_events": split, "peak_source": f"hbm_gbs of {src}"}
    # the same seven weights loaded in bf16 (2 B read per weight)
    wb = [(label, W.to(torch.bfloat16), w) for label, W, w in weights]
    for _ in range(2):
        for _, Wb, w in wb:
            q.quantize_nf4(Wb, out=w, workspace=ws)
    torch.cuda.synchronize()
    a.record()
    for _ in range(reps):
        for _, Wb, w in wb:
            q.quantize_nf4(Wb, out=w, workspace=ws)
    b.record()
    torch.cuda.synchronize()
    tb = a.elapsed_time(b) / reps
    qbytes_b = sum(workloads.quant_bytes(*Wb.shape) - 2 * Wb.numel() for _, Wb, _ in wb)
    out["quantize_bf16_65b_layer"] = {"ms": tb, "GB/s": qbytes_b / (tb * 1e-3) / 1e9,
                                      "frac_hbm": qbytes_b / (tb * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                      "bytes_per_weight": 2.516}
    del wb
    # NF4 vs the uniform INT4 code: round-trip error on normal and Student-t weights (same kernels)
    cmp = {}
    for dist in ("normal", "student_t5"):
        W = synth.weight(4096, 4096, 0.02, dist, seed=21).to(dev)
        wn = q.quantize_nf4(W)
        w4 = q.quantize_codebook(W, q.CODEBOOK_INT4)
        en = float((q.dequantize_nf4(wn).float() - W).norm() / W.norm())
        e4 = float((q.dequantize_codebook(w4, q.CODEBOOK_INT4).float() - W).norm() / W.norm())
        cmp[dist] = {"nf4_rel_error": en, "int4_rel_error": e4, "int4_over_nf4": e4 / en}
    torch.cuda.synchronize()
    a.record()
    for _ in range(reps):
        for _, W, w in weights:
            q.quantize_codebook(W, q.CODEBOOK_INT4, out=w, workspace=ws)
    b.record()
    torch.cuda.synchronize()
    t4 = a.elapsed_time(b) / reps
    cmp["int4_quantize_65b_layer"] = {"ms": t4, "frac_hbm": qbytes / (t4 * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    out["nf4_vs_int4_7b_attn"] = cmp
    deq_out = [torch.empty(w.rows, w.cols, dtype=torch.bfloat16, device=dev) for _, _, w in weights]
    for (_, _, w), o in zip(weights, deq_out):
        q.dequantize_nf4(w, out=o)
    torch.cuda.synchronize()
    a.record()
    for _ in range(reps):
        for (_, _, w), o in zip(weights, deq_out):
            q.dequantize_nf4(w, out=o)
    b.record()
    torch.cuda.synchronize()
    tot = a.elapsed_time(b) / reps
    dbytes = sum(workloads.gemv_weight_bytes(w.rows, w.cols) + 2 * w.rows * w.cols for _, _, w in weights)
    out["dequantize_65b_layer"] = {"ms": tot, "GB/s": dbytes / (tot * 1e-3) / 1e9,
                                   "frac_hbm": dbytes / (tot * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    del deq_out, weights, ws
    torch.cuda.empty_cache()
    return out


def comp_dropout(q, dev, peaks, n=50):
    """fwd+bwd of the 7B attention projection with LoRA dropout p = 0.05 (the
    pages' setting; keep mask drawn on the host), against the same step
    without dropout; same FLOP count."""
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    a, b = ev(), ev()
    M, n_in, n_out, r, alpha, p = 4096, 4096, 4096, 16, 32.0, 0.05
    prob = synth.problem(M, n_in, n_out, r, seed=4)
    w = q.quantize_nf4(prob["W"].to(dev))
    x, A, B, dh = (prob[k].to(dev) for k in ("x", "A", "B", "dh"))
    keep = torch.from_numpy(np.random.default_rng(4).random((M, n_in)) >= p).to(dev)
    kb = q.pack_keep_mask(keep)
    res = {}
    for label, fwd, bwd in (("plain", lambda: q.linear_fwd(x, w, A, B, alpha),
                             lambda us: q.linear_bwd(dh, x, us, w, A, B, alpha)),
                            ("dropout_p0.05", lambda: q.linear_fwd_dropout(x, w, A, B, alpha, kb, p),
                             lambda us: q.linear_bwd_dropout(dh, x, us, w, A, B, alpha, kb, p))):
        for _ in range(3):
            _, us = fwd()
            bwd(us)
        torch.cuda.synchronize()
        a.record()
        for _ in range(n):
            _, us = fwd()
            bwd(us)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / n
        q.timing_reset()                            # the same steps again, kernels bracketed by events
        q.timing_enable(True)
        for _ in range(n):
            _, us = fwd()
            bwd(us)
        torch.cuda.synchronize()
        q.timing_enable(False)
        kern = {}
        for name in q.KERNEL_NAMES:
            t, k = q.timing_collect(name)
            if k:
                kern[name] = 1e3 * t / n
        res[label] = {"ms": ms, "TFLOP/s": workloads.fwd_bwd_flops(M, n_in, n_out, r) / (ms * 1e-3) / 1e12,
                      "kernel_us_per_step": kern}
    res["dropout_overhead"] = res["dropout_p0.05"]["ms"] / res["plain"]["ms"] - 1.0
    return {"lora_dropout_llama7b_attn": res}


def dropout_steps_once(q, dev, steps=2):
    """Untimed LoRA-dropout steps of the 7B attention projection (p = 0.05),
    for a profiler's capture of the masked kernels alone."""
    M, n_in, n_out, r, alpha, p = 4096, 4096, 4096, 16, 32.0, 0.05
    prob = synth.problem(M, n_in, n_out, r, seed=4)
    w = q.quantize_nf4(prob["W"].to(dev))
    x, A, B, dh = (prob[k].to(dev) for k in ("x", "A", "B", "dh"))
    keep = torch.from_numpy(np.random.default_rng(4).random((M, n_in)) >= p).to(dev)
    kb = q.pack_keep_mask(keep)
    for _ in range(1 + steps):
        _, us = q.linear_fwd_dropout(x, w, A, B, alpha, kb, p)
        q.linear_bwd_dropout(dh, x, us, w, A, B, alpha, kb, p)
    torch.cuda.synchronize()
    return {"ok": q.last_device_status() == 0, "steps": 1 + steps}


def comp_merge(q, dev, peaks, src, reps=5):
    """Adapter merge into a bf16 base and its lossy re-quantization to NF4, on
    the 7B attention projection (r=16) and the 65B down projection (r=64).
    Merge bytes: packed weight read + bf16 written (2.516 B/weight); the loss
    is the relative Frobenius error of the re-quantized merged weight."""
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    a, b = ev(), ev()
    res = {}
    for label, n_out, n_in, r, alpha, std in (("llama7b-attn-4096x4096-r16", 4096, 4096, 16, 32.0, 0.02),
                                              ("llama65b-down-22016x8192-r64", 8192, 22016, 64, 16.0, 0.01)):
        W = synth.weight(n_out, n_in, std, seed=3).to(dev)
        A = synth.lora_A(r, n_in).to(dev)
        B = (synth.lora_B(n_out, r).float() * 10).to(torch.bfloat16).to(dev)   # a trained-size adapter
        w = q.quantize_nf4(W)
        merged = torch.empty(n_out, n_in, dtype=torch.bfloat16, device=dev)
        w2 = q.alloc_nf4(n_out, n_in, dev)
        for _ in range(2):
            q.merge_adapter(w, A, B, alpha, out=merged)
            q.quantize_nf4(merged, out=w2)
        torch.cuda.synchronize()
        a.record()
        for _ in range(reps):
            q.merge_adapter(w, A, B, alpha, out=merged)
        b.record()
        torch.cuda.synchronize()
        t_merge = a.elapsed_time(b) / reps
        a.record()
        for _ in range(reps):
            q.quantize_nf4(merged, out=w2)
        b.record()
        torch.cuda.synchronize()
        t_req = a.elapsed_time(b) / reps
        mbytes = workloads.gemv_weight_bytes(n_out, n_in) + 2 * n_out * n_in
        qbytes = n_out * n_in * (2 + 0.5 + 1 / 64) + 4 * (n_out * n_in // 64 // 256)
        base_f = q.dequantize_nf4(w).float()
        req_f = q.dequantize_nf4(w2).float()
        mf = merged.float()
        res[f"merge_{label}"] = {
            "merge_ms": t_merge, "merge_GB/s": mbytes / (t_merge * 1e-3) / 1e9,
            "merge_frac_hbm": mbytes / (t_merge * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "requantize_bf16_ms": t_req, "requantize_GB/s": qbytes / (t_req * 1e-3) / 1e9,
            "requantize_frac_hbm": qbytes / (t_req * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "merge_into_4bit_rel_error": float((req_f - mf).norm() / mf.norm()),
            "base_quantization_rel_error": float((base_f - W).norm() / W.norm()),
            "adapter_update_rel_size": float((mf - base_f).norm() / base_f.norm()),
            "peak_source": f"hbm_gbs of {src}"}
        del W, w, w2, merged, base_f, req_f, mf
        torch.cuda.empty_cache()
    return res


def comp_gemv(q, dev, peaks, n=60):
    """Few-token forward on the 70B MLP shapes; 3 weight copies (3 x 121 MB > L2)."""
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    a, b = ev(), ev()
    g = workloads.GEMV_70B
    gres = {}
    for (label, n_in, n_out) in g.projections:
        ws_list = []
        for i in range(3):
            W = synth.weight(n_out, n_in, g.w_std, seed=10 + i).to(dev)
            ws_list.append(q.quantize_nf4(W))
            del W
        A = synth.lora_A(g.r, n_in).to(dev)
        B = synth.lora_B(n_out, g.r).to(dev)
        for M in g.M:
            x = synth.activations(M, n_in, seed=M).to(dev)
            h = torch.empty(M, n_out, dtype=torch.bfloat16, device=dev)
            us = torch.empty(M, g.r, dtype=torch.bfloat16, device=dev)
            wsf = torch.empty(max(1, q.workspace_size(q.OP_LINEAR_FWD, M, n_in, n_out, g.r)), dtype=torch.uint8,
                              device=dev)
            call = lambda i: q.linear_fwd(x, ws_list[i % 3], A, B, g.alpha, h=h, us=us, workspace=wsf)  # noqa: E731
            for i in range(3):
                call(i)
            torch.cuda.synchronize()
            a.record()                                  # whole calls, no per-kernel events
            for i in range(n):
                call(i)
            b.record()
            torch.cuda.synchronize()
            call_ms = a.elapsed_time(b) / n
            q.timing_reset()                            # the same calls again, kernels bracketed by events
            q.timing_enable(True)
            for i in range(n):
                call(i)
            torch.cuda.synchronize()
            q.timing_enable(False)
            kms, kn = q.timing_collect("gemv")
            parts = {}
            for name in ("lora_fewtok", "lora_rowwise", "gemv", "gemv_finalize", "lora_pad"):
                t_, n_ = q.timing_collect(name)
                if n_:
                    parts[name] = 1e3 * t_ / n
            # the same three calls captured once in a CUDA graph and replayed:
            # the device time of a call without the host's per-call work
            try:
                side = torch.cuda.Stream()
                side.wait_stream(torch.cuda.current_stream())
                with torch.cuda.stream(side):
                    for i in range(3):
                        call(i)
                torch.cuda.current_stream().wait_stream(side)
                torch.cuda.synchronize()
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    for i in range(3):
                        call(i)
                graph.replay()
                torch.cuda.synchronize()
                reps = max(1, n // 3)
                a.record()
                for _ in range(reps):
                    graph.replay()
                b.record()
                torch.cuda.synchronize()
                graph_us = 1e3 * a.elapsed_time(b) / (3 * reps)
                del graph
            except Exception as e:              # report, do not fail the benchmark
                graph_us = f"capture failed: {type(e).__name__}: {e}"[:200]
            wbytes = workloads.gemv_weight_bytes(n_out, n_in)
            gres[f"{label}_{n_in}x{n_out}_M{M}"] = {
                "call_us": 1e3 * call_ms, "gemv_kernel_us": 1e3 * kms / kn if kn else None,
                "graph_replay_call_us": graph_us,
                "packed_weight_GB/s_call": wbytes / (call_ms * 1e-3) / 1e9,
                "frac_hbm_call": wbytes / (call_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "packed_weight_GB/s_kernel": wbytes / (kms / kn * 1e-3) / 1e9 if kn else None,
                "frac_hbm_kernel": (wbytes / (kms / kn * 1e-3) / 1e9 / peaks["hbm_gbs"]) if kn else None,
                "kernel_us_per_call": parts}
        del ws_list
        torch.cuda.empty_cache()
    return {"gemv_70b": gres}


def comp_workloads(q, dev, peaks, n=10):
    """fwd+bwd of the 7B attention projection and of the 7B MLP (3 projections),
    each projection on its own inputs, clean CUDA-event timing."""
    out = {}
    for wl in (workloads.ATTN_7B, workloads.MLP_7B):
        L = LayerState(q, wl, 0, dev)
        for _ in range(3):
            L.step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n):
            L.step()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / n
        tf = L.flops() / (ms * 1e-3) / 1e12
        out[wl.name] = {"ms": ms, "TFLOP/s": tf, "frac_bf16_burst": tf / peaks["bf16_tflops"],
                        "frac_bf16_sustained": tf / peaks["bf16_tflops_sustained"]}
        del L
        torch.cuda.empty_cache()
    return out


def layer_step_once(q, dev, projections=None, steps=1):
    """Untimed steps of the headline layer, or of some of its projections
    (for a profiler's launch list or a capture on a smaller device footprint)."""
    wl = WL
    if projections is not None:
        import dataclasses
        wl = dataclasses.replace(WL, projections=tuple(WL.projections[i] for i in projections))
    L = LayerState(q, wl, 0, dev)
    L.step()
    torch.cuda.synchronize()
    q.timing_reset()
    q.timing_enable(True)
    for _ in range(steps):
        L.step()
    torch.cuda.synchronize()
    q.timing_enable(False)
    kern = {}
    for name in q.KERNEL_NAMES:
        t, n = q.timing_collect(name)
        if n:
            kern[name] = {"avg_us": 1e3 * t / n, "launches": n}
    return {"ok": q.last_device_status() == 0, "projections": [p[0] for p in wl.projections], "steps": steps,
            "kernels": kern}


def components(q, dev, only=None):
    """Extra measurements outside the timed region: quantizer and dequantizer
    HBM throughput, the few-token GEMV, and the other fwd+bwd workloads."""
    peaks, src = load_peaks()
    out = {}
    if only in (None, "quantize"):
        out.update(comp_quantize(q, dev, peaks, src))
    if only in (None, "gemv"):
        out.update(comp_gemv(q, dev, peaks))
    if only in (None, "workloads"):
        out.update(comp_workloads(q, dev, peaks))
    if only in (None, "merge"):
        out.update(comp_merge(q, dev, peaks, src))
    if only in (None, "dropout"):
        out.update(comp_dropout(q, dev, peaks))
    if only == "layer_step":
        out.update(layer_step_once(q, dev))
    if only == "q_proj_steps":
        out.update(layer_step_once(q, dev, projections=(0,), steps=4))
    if only == "dropout_steps":
        out.update(dropout_steps_once(q, dev))
    return out


# ---------------------------------------------------------------------------- main
def main():
    args = parse()
    if args.impl == "reference":
        # the oracle arm runs on the host cores of rank 0 only: no device, no process group
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if world != args.gpus:
            raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_setup(args)
    try:
        if args.only is not None:
            import bit_nf4_quantized_11_b200 as q
            q.load()
            if rank == 0:
                print(json.dumps({"only": args.only,
                                  "components": components(q, torch.device("cuda", local), args.only)}), flush=True)
            return
        line = run_ours(args, world, rank, local)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
        elif rank == 0:
            line["cpu_baseline"] = None
        if rank == 0 and world == 1 and not args.no_components:
            import bit_nf4_quantized_11_b200 as q
            line["components"] = components(q, torch.device("cuda", local))
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
