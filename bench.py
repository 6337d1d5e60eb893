#!/usr/bin/env python
"""bench.py -- the grouped NF4 W4A16 expert GEMM hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  moe_align (token->expert sort of topk_ids) -> grouped NF4 GEMM gate_up
  (fused SwiGLU where the workload has it) -> grouped NF4 GEMM down,
with sizes/expert_ids handed from the sort to the GEMMs on the device.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload mixtral_8x22b|olmoe|tiny|qwen3_30b_a3b|gpt_oss_120b]
                    [--only]

Prints ONE JSON line on rank 0. The headline workload (default: the
Mixtral-8x22B-shaped prefill, the largest single-GPU configuration) is timed
for exactly K steps; `value` is its whole-job throughput (all ranks) of the
metric: TFLOP/s for the prefill workload (2*M*N*K per GEMM), HBM GB/s for the
decode workloads (algorithmic bytes: touched expert weights + absmax + x + y +
sort I/O). On one GPU the other four configurations follow (unless --only),
each with its own step throughput, per-GEMM roofline and oracle baseline under
"configs". With N > 1 every rank runs an independent replica of the headline
(the path does not shard; weak scaling), the timed region is bracketed by a
barrier + synchronize and its time is the max over ranks.

Timing: CUDA events on the launching stream. Each step is a CUDA graph of the
C-ABI calls (they are capture-safe: no host sync, no allocation). Weight
stacks rotate over enough replicas that a step never finds its weights in
L2. Per-kernel durations for the roofline come from external event nodes
captured inside the step graphs (the last replay of each replica's graph).
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import re
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "grouped NF4 GEMM: HBM GB/s & % roofline (decode); TFLOPS & % peak (prefill)"
L2_BYTES = 126 * 1024 * 1024
DEFAULT_STEPS = {"tiny": 20000, "olmoe": 20000, "qwen3_30b_a3b": 5000, "gpt_oss_120b": 500,
                 "mixtral_8x22b": 150}


# ----------------------------------------------------------------- helpers
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def source_hash(path):
    """sha256 prefix of a kernel source's code: comments, trailing blanks and
    empty lines removed (they do not change what the compiler emits), so a
    comment edit keeps the committed counters valid and a code edit does not."""
    src = open(path, encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    code = "\n".join(line.rstrip() for line in src.splitlines() if line.strip())
    return hashlib.sha256(code.encode("utf-8")).hexdigest()[:16]


def traffic_for(kernel, workload, gemm):
    """DRAM bytes per launch from the committed ncu summary, or None if the
    kernel source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(path))
        ent = d[kernel][f"{workload}.{gemm}"]
        src = os.path.join(ROOT, "grouped_nf4_w4a16_b200", "csrc", ent["source"])
        if source_hash(src) != ent["source_sha256"]:
            return None
        return float(ent["dram_bytes_per_launch"])
    except Exception:
        return None


class Clocks:
    """nvidia-smi sampler (clocks and throttle reasons) around a region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if ts < t0 or ts > t1:
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def _cuda_driver():
    lib = ctypes.CDLL("libcuda.so.1")
    lib.cuEventRecordWithFlags.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint]
    lib.cuEventRecordWithFlags.restype = ctypes.c_int
    lib.cuEventElapsedTime.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_void_p,
                                       ctypes.c_void_p]
    lib.cuEventElapsedTime.restype = ctypes.c_int
    lib.cuEventCreate.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_uint]
    lib.cuEventCreate.restype = ctypes.c_int
    lib.cuGraphGetNodes.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_size_t)]
    lib.cuGraphGetNodes.restype = ctypes.c_int
    lib.cuGraphNodeGetType.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int)]
    lib.cuGraphNodeGetType.restype = ctypes.c_int
    lib.cuGraphKernelNodeGetParams = getattr(lib, "cuGraphKernelNodeGetParams_v2",
                                             lib.cuGraphKernelNodeGetParams)
    lib.cuGraphKernelNodeGetParams.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    lib.cuGraphKernelNodeGetParams.restype = ctypes.c_int
    lib.cuFuncGetName.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.c_void_p]
    lib.cuFuncGetName.restype = ctypes.c_int
    return lib


def _new_event(drv):
    """A timing-enabled CUevent created through the driver API."""
    ev = ctypes.c_void_p(0)
    st = drv.cuEventCreate(ctypes.byref(ev), 0)
    if st != 0:
        raise RuntimeError(f"cuEventCreate failed with CUresult {st}")
    return ev


def _elapsed_ms(drv, a, b):
    """Elapsed time between two events recorded by external graph nodes, or
    NaN when the driver has no timestamps for them (e.g. under a profiler that
    replays graph nodes one by one)."""
    out = ctypes.c_float(0.0)
    st = drv.cuEventElapsedTime(ctypes.byref(out), a, b)
    if st != 0:
        return float("nan")
    return float(out.value)


def max_over_ranks(x, world, device):
    """The largest value of x over all ranks (x itself when world == 1). Every
    rank must call it at the same point: it is one all-reduce."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ problem
class HostProblem:
    """Seeded synthetic inputs of one workload as host arrays, with the
    algorithmic work per step. Imports nothing from the product library, so
    the reference arm (the oracle on the host cores) never loads it."""

    def __init__(self, name, seed=0):
        self.w = synth.WORKLOADS[name]
        w = self.w
        self.name = name
        self.topk_np = synth.routing(w, seed)
        self.U = int(np.unique(self.topk_np).size)
        self.gemms = []
        touched_bytes = 0
        for g in w.gemms:
            packed, absmax = synth.random_packed_stack(w.E, g.N, g.K, seed=seed, which=g.name)
            x = synth.activations_bf16(w.M, g.K, seed=seed, which=g.name)
            n_out = g.N // 2 if g.swiglu else g.N
            self.gemms.append(dict(
                g=g, packed_np=packed, absmax_np=absmax, x_np=x, n_out=n_out,
                bytes=self.U * g.N * g.K * 9 // 16 + w.M * g.K * 2 + w.M * n_out * 2,
                flops=2 * w.M * g.N * g.K))
            touched_bytes += self.U * g.N * g.K * 9 // 16
        # weight-stack replicas rotated per step so that a step never finds its
        # weights in L2 (none needed when a step touches more than 2x L2)
        self.R = (1 if touched_bytes > 2 * L2_BYTES
                  else 1 + -(-int(1.5 * L2_BYTES) // touched_bytes))
        S = w.T * w.top_k
        self.align_bytes = S * 4 + S * 4 + 2 * w.E * 4 + 4
        self.step_bytes = self.align_bytes + sum(d["bytes"] for d in self.gemms)
        self.step_flops = sum(d["flops"] for d in self.gemms)
        self.prefill = w.regime == "prefill"

    def describe(self):
        w = self.w
        return {
            "workload": f"{w.name}: {w.description}",
            "E": w.E, "top_k": w.top_k, "tokens": w.T, "rows": w.M,
            "gemms": [f"{d['g'].name} K={d['g'].K} N={d['g'].N}" + (" +SwiGLU" if d['g'].swiglu else "")
                      for d in self.gemms],
            "touched_experts": self.U,
            "weights": "uniform random NF4 codes, absmax U[0.04,0.06] (values do not affect timing)",
            "l2": (f"{self.R} weight-stack replicas rotated per step "
                   f"(touched bytes of the other replicas > L2)" if self.R > 1 else
                   "touched weights per step > 2x L2 (no replica needed)"),
        }


class Problem(HostProblem):
    """HostProblem plus its device tensors and the step's C-ABI calls."""

    def __init__(self, name, seed=0, device="cuda"):
        super().__init__(name, seed)
        w = self.w
        self.device = device
        import grouped_nf4_w4a16_b200 as gnf4
        self.gnf4 = gnf4
        self.topk = torch.from_numpy(self.topk_np).to(device)
        S = w.T * w.top_k
        self.sorted_idx = torch.empty(S, dtype=torch.int32, device=device)
        self.sizes = torch.empty(w.E, dtype=torch.int32, device=device)
        self.expert_ids = torch.empty(w.E, dtype=torch.int32, device=device)
        self.num_groups = torch.empty(1, dtype=torch.int32, device=device)
        self.ws_align = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_MOE_ALIGN, S, E=w.E), device)
        for d in self.gemms:
            g = d["g"]
            wd = torch.from_numpy(d["packed_np"]).to(device)
            ad = torch.from_numpy(d["absmax_np"]).to(device)
            d["W"] = [wd] + [wd.clone() for _ in range(self.R - 1)]
            d["A"] = [ad] + [ad.clone() for _ in range(self.R - 1)]
            d["x"] = torch.from_numpy(d["x_np"].view(np.int16)).to(device).view(torch.bfloat16)
            d["y"] = torch.empty((w.M, d["n_out"]), dtype=torch.bfloat16, device=device)
            d["ws"] = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(
                gnf4.GNF4_OP_GROUPED_GEMM, w.M, g.N, g.K, w.E, w.E), device)
            d["epi"] = gnf4.GNF4_EPI_SWIGLU if g.swiglu else gnf4.GNF4_EPI_NONE

    def launch(self, r, events=None, drv=None, stream=None):
        """Enqueue one step with weight replica r (optionally recording events)."""
        gnf4 = self.gnf4

        def ev(i):
            if events is not None:
                # CU_EVENT_RECORD_EXTERNAL: a real timestamp node inside the graph
                st = drv.cuEventRecordWithFlags(events[i], ctypes.c_void_p(stream.cuda_stream), 1)
                if st != 0:
                    raise RuntimeError(f"cuEventRecordWithFlags failed with CUresult {st}")
        ev(0)
        gnf4.gnf4_moe_align(self.topk, self.w.E, sorted_idx=self.sorted_idx, sizes=self.sizes,
                            expert_ids=self.expert_ids, num_groups=self.num_groups,
                            workspace=self.ws_align)
        ev(1)
        for i, d in enumerate(self.gemms):
            gnf4.gnf4_grouped_gemm(d["x"], d["W"][r], d["A"][r], self.sizes, self.expert_ids,
                                   epilogue=d["epi"], y=d["y"], workspace=d["ws"])
            ev(2 + i)

    def free(self):
        for d in self.gemms:
            for k in ("W", "A", "x", "y", "ws"):
                d.pop(k, None)


def graph_kernels(drv, graph):
    """Names of the kernel nodes of a captured (kept) CUDA graph."""
    n = ctypes.c_size_t(0)
    h = ctypes.c_void_p(graph.raw_cuda_graph())
    if drv.cuGraphGetNodes(h, None, ctypes.byref(n)) != 0:
        return None
    nodes = (ctypes.c_void_p * n.value)()
    if drv.cuGraphGetNodes(h, nodes, ctypes.byref(n)) != 0:
        return None
    names = []
    for i in range(n.value):
        t = ctypes.c_int(-1)
        if drv.cuGraphNodeGetType(ctypes.c_void_p(nodes[i]), ctypes.byref(t)) != 0:
            return None
        if t.value != 0:          # CU_GRAPH_NODE_TYPE_KERNEL
            continue
        params = (ctypes.c_byte * 256)()   # CUDA_KERNEL_NODE_PARAMS (v2); func first
        if drv.cuGraphKernelNodeGetParams(ctypes.c_void_p(nodes[i]), params) != 0:
            names.append("?")
            continue
        func = ctypes.c_void_p.from_buffer(params).value
        nm = ctypes.c_char_p()
        ok = drv.cuFuncGetName(ctypes.byref(nm), ctypes.c_void_p(func)) == 0 and nm.value
        names.append(nm.value.decode() if ok else "?")
    return names


# --------------------------------------------------------------- our arm
def run_ours(name, steps, warmup, world, dev, stream, drv, with_e2e=True):
    """Capture, warm up and time `steps` steps of workload `name`. Returns a
    dict with the Problem, the timed ms (max over ranks), per-kernel ms, the
    clocks seen, the end-to-end timing and the kernels of one step graph."""
    prob = Problem(name, seed=0, device=dev)
    nk = 1 + len(prob.gemms)
    # Per weight replica: a plain step graph (timed; consecutive kernels keep
    # their programmatic launch edges) and a copy with external event nodes
    # around each C-ABI call (per-call durations, replayed after the timing).
    graphs, ev_graphs, evs = [], [], []
    with torch.cuda.stream(stream):
        for r in range(prob.R):      # eager warm-up (sets kernel attributes, first-call work)
            prob.launch(r)
        torch.cuda.synchronize()
        for r in range(prob.R):
            g = torch.cuda.CUDAGraph(keep_graph=True)
            with torch.cuda.graph(g, stream=stream):
                prob.launch(r)
            g.instantiate()
            graphs.append(g)
            e = [_new_event(drv) for _ in range(nk + 1)]
            ge = torch.cuda.CUDAGraph()
            with torch.cuda.graph(ge, stream=stream):
                prob.launch(r, events=e, drv=drv, stream=stream)
            ev_graphs.append(ge)
            evs.append(e)
    torch.cuda.synchronize()
    step_kernels = graph_kernels(drv, graphs[0])

    clocks = Clocks(dev.index if dev.index is not None else 0)
    clocks.start()
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        for i in range(warmup):
            graphs[i % prob.R].replay()
        # keep the GPU busy for ~0.5 s before timing so clocks settle
        t_end = time.time() + 0.5
        i = 0
        while time.time() < t_end:
            graphs[i % prob.R].replay()
            i += 1
    stream.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    start.record(stream)
    with torch.cuda.stream(stream):
        for i in range(steps):
            graphs[i % prob.R].replay()
    stop.record(stream)
    stop.synchronize()
    t1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ms = start.elapsed_time(stop)
    # clock window: if the timed region was short, keep replaying the same
    # steps for ~1 s so the sampler sees this workload under load
    if t1 - t0 < 1.0:
        with torch.cuda.stream(stream):
            t_end = time.time() + 1.0
            i = 0
            while time.time() < t_end:
                graphs[i % prob.R].replay()
                i += 1
        stream.synchronize()
    t2 = time.time()
    clk = clocks.stop(t0, t2)

    # per-call durations: external event nodes of the last of a few replays
    # of each replica's instrumented graph (calls serialised by the nodes)
    with torch.cuda.stream(stream):
        for _ in range(3):
            for ge in ev_graphs:
                ge.replay()
    stream.synchronize()
    per_kernel = [[] for _ in range(nk)]
    for e in evs:
        for k in range(nk):
            per_kernel[k].append(_elapsed_ms(drv, e[k], e[k + 1]))
    kern_ms = [sum(v) / len(v) for v in per_kernel]   # NaN if a timestamp was missing

    ms = max_over_ranks(ms, world, dev)
    e2e = None
    if with_e2e:
        # host (pinned) inputs -> device, the C-ABI calls, results -> host
        e2e = run_e2e(prob, stream, max(3, min(steps, 2000) // 10))
        e2e = (max_over_ranks(e2e[0], world, dev),) + tuple(e2e[1:])
    del graphs, ev_graphs
    return dict(prob=prob, ms=ms, kern_ms=kern_ms, clocks=clk, e2e=e2e,
                step_kernels=step_kernels, steps=steps, warmup=warmup)


def roofline(prob, d, k_ms, pk):
    """Roofline of one GEMM launch: algorithmic bytes (decode, HBM-bound) or
    FLOPs (prefill, tensor-bound) per launch over its event-timed duration."""
    kernel = "prefill_gemm_kernel" if prob.prefill else "decode_gemm_kernel"
    if prob.prefill:
        # timed inside seconds of back-to-back steps: the sustained bf16 figure
        achieved = d["flops"] / (k_ms / 1e3) / 1e12
        peak, which = pk["bf16_tflops_sustained"], "bf16_tflops_sustained"
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "frac_of_nominal_2250": achieved / 2250.0}
    else:
        achieved = d["bytes"] / (k_ms / 1e3) / 1e9
        peak, which = pk["hbm_gbs"], "hbm_gbs"
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak}
    roof["traffic"] = traffic_for(kernel.replace("_kernel", "") if prob.prefill else kernel,
                                  prob.name, d["g"].name)
    roof["kernel"] = f"{kernel} ({d['g'].name} launch)"
    roof["algorithmic_per_launch"] = d["flops"] if prob.prefill else d["bytes"]
    roof["launch_ms"] = k_ms
    roof["peak_source"] = (f"measured {which} (MEASURED_PEAKS.json)" if pk["source"] == "measured"
                           else f"fallback {which}")
    return roof


def kernels_entry(prob, kern_ms):
    kernels = {"moe_align": {"ms": kern_ms[0]}}
    for i, d in enumerate(prob.gemms):
        entry = {"ms": kern_ms[1 + i], "GB/s": d["bytes"] / (kern_ms[1 + i] / 1e3) / 1e9}
        if prob.prefill:
            entry["TFLOP/s"] = d["flops"] / (kern_ms[1 + i] / 1e3) / 1e12
        kernels[d["g"].name] = entry
    return kernels


def time_glue(prob, stream, reps=50):
    """The entry points beside the GEMMs, timed outside the step: the router's
    top-k on seeded N(0,1) logits [T, E], the weighted combine of the last
    GEMM's output [T*top_k, H] and, for decode workloads, the dgrad of the last
    GEMM with that output as dy. CUDA events around `reps` back-to-back
    launches after a warm-up; the inputs stay in L2 between launches."""
    gnf4 = prob.gnf4
    w = prob.w
    dev = prob.topk.device
    rng = np.random.default_rng(1)
    logits = torch.from_numpy(rng.standard_normal((w.T, w.E)).astype(np.float32)).to(dev)
    ids = torch.empty((w.T, w.top_k), dtype=torch.int32, device=dev)
    wts = torch.empty((w.T, w.top_k), dtype=torch.float32, device=dev)
    y = prob.gemms[-1]["y"]
    H = y.shape[1]
    out = torch.empty((w.T, H), dtype=torch.bfloat16, device=dev)
    ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_MOE_COMBINE, w.T * w.top_k), dev)
    S = w.T * w.top_k
    calls = {
        "router_topk": (lambda: gnf4.gnf4_router_topk(logits, w.top_k, renormalize=True,
                                                      topk_ids=ids, topk_weights=wts),
                        w.T * w.E * 4 + S * 8),
        "combine": (lambda: gnf4.gnf4_moe_combine(y, prob.sorted_idx, wts, out=out, workspace=ws),
                    S * H * 2 + w.T * H * 2 + S * 8),
    }
    if not prob.prefill:
        # the dgrad of the last GEMM (tensor-core kernel for decode-sized batches)
        d = prob.gemms[-1]
        g = d["g"]
        dx = torch.empty((w.M, g.K), dtype=torch.bfloat16, device=dev)
        ws_dg = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_GROUPED_DGRAD, w.M, g.N,
                                                              g.K, w.E, w.E), dev)
        calls["dgrad"] = (lambda: gnf4.gnf4_grouped_dgrad(y, d["W"][0], d["A"][0], prob.sizes,
                                                          prob.expert_ids, dx=dx, workspace=ws_dg),
                          prob.U * g.N * g.K * 9 // 16 + w.M * g.N * 2 + w.M * g.K * 2)
    res = {}
    with torch.cuda.stream(stream):
        for name, (fn, nbytes) in calls.items():
            for _ in range(5):
                fn()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b.record(stream)
            b.synchronize()
            ms = a.elapsed_time(b) / reps
            res[name] = {"ms": ms, "bytes": nbytes, "GB/s": nbytes / (ms / 1e3) / 1e9}
    res["how"] = (f"outside the timed step; {reps} back-to-back launches per entry point "
                  f"(router: T x E fp32 logits; combine: T*top_k x {H} bf16 rows; dgrad of the last "
                  f"GEMM, decode workloads only), inputs L2-resident")
    return res


def run_e2e(prob, stream, steps):
    """The step through the public entry points with host inputs and
    outputs: every step copies its inputs in from pinned host memory and its
    results out to pinned host memory. Pipelined as a serving loop runs it:
    step i's inputs are copied in (one copy stream) and step i-1's results
    copied out (another) while step i-1 / i computes, over two sets of device
    buffers; the timed region runs from the first copy in to the last copy
    out."""
    gnf4 = prob.gnf4
    dev = prob.topk.device
    h_topk = torch.from_numpy(prob.topk_np).pin_memory()
    h_x = [torch.from_numpy(d["x_np"].view(np.int16)).pin_memory() for d in prob.gemms]
    h_y = [torch.empty(d["y"].shape, dtype=torch.int16).pin_memory() for d in prob.gemms]
    nbuf = 2
    d_topk = [torch.empty_like(prob.topk) for _ in range(nbuf)]
    d_x = [[torch.empty(d["x"].shape, dtype=torch.int16, device=dev) for d in prob.gemms]
           for _ in range(nbuf)]
    d_y = [[torch.empty_like(d["y"]) for d in prob.gemms] for _ in range(nbuf)]
    h2d = h_topk.numel() * 4 + sum(t.numel() * 2 for t in h_x)
    d2h = sum(t.numel() * 2 for t in h_y)
    copy_in = torch.cuda.Stream(device=dev)
    copy_out = torch.cuda.Stream(device=dev)
    in_ready = [torch.cuda.Event() for _ in range(nbuf)]
    computed = [torch.cuda.Event() for _ in range(nbuf)]
    out_done = [torch.cuda.Event() for _ in range(nbuf)]

    def one(i, r):
        j = i % nbuf
        with torch.cuda.stream(copy_in):
            if i >= nbuf:
                copy_in.wait_event(computed[j])     # buffer j's inputs read by step i - 2
            d_topk[j].copy_(h_topk, non_blocking=True)
            for a, b in zip(d_x[j], h_x):
                a.copy_(b, non_blocking=True)
            in_ready[j].record(copy_in)
        with torch.cuda.stream(stream):
            stream.wait_event(in_ready[j])
            if i >= nbuf:
                stream.wait_event(out_done[j])      # buffer j's results copied out by step i - 2
            gnf4.gnf4_moe_align(d_topk[j], prob.w.E, sorted_idx=prob.sorted_idx,
                                sizes=prob.sizes, expert_ids=prob.expert_ids,
                                num_groups=prob.num_groups, workspace=prob.ws_align)
            for k, d in enumerate(prob.gemms):
                gnf4.gnf4_grouped_gemm(d_x[j][k].view(torch.bfloat16), d["W"][r], d["A"][r],
                                       prob.sizes, prob.expert_ids, epilogue=d["epi"],
                                       y=d_y[j][k], workspace=d["ws"])
            computed[j].record(stream)
        with torch.cuda.stream(copy_out):
            copy_out.wait_event(computed[j])
            for k in range(len(prob.gemms)):
                h_y[k].copy_(d_y[j][k].view(torch.int16), non_blocking=True)
            out_done[j].record(copy_out)

    for i in range(3):
        one(i, i % prob.R)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(copy_in)
    for i in range(steps):
        one(i, i % prob.R)
    b.record(copy_out)
    b.synchronize()
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / steps
    return ms, h2d, d2h, steps


# -------------------------------------------------------- oracle (CPU) arm
def oracle_step_sample(prob, budget_s):
    """Time the CPU oracle on a bounded sample of the step. Returns
    (seconds per full step, description, threads)."""
    import oracle
    w = prob.w
    nthreads = oracle.num_threads()
    t_align = time.perf_counter()
    _, sizes, experts, _ = oracle.moe_align(prob.topk_np, w.E)
    t_align = time.perf_counter() - t_align
    # rows per GEMM: all rows if a full step fits the budget, else a row sample
    per_row = []
    for d in prob.gemms:
        rows = np.array([0, w.M - 1])
        t = time.perf_counter()
        oracle.grouped_gemm_f64(d["x_np"], d["packed_np"], d["absmax_np"], sizes, experts, rows=rows)
        per_row.append((time.perf_counter() - t) / rows.size)
    full_est = t_align + sum(per_row) * w.M
    if full_est <= budget_s / 3:
        n = 0
        t = time.perf_counter()
        while True:
            oracle.moe_align(prob.topk_np, w.E)
            for d in prob.gemms:
                y = oracle.grouped_gemm_f64(d["x_np"], d["packed_np"], d["absmax_np"], sizes, experts)
                if d["g"].swiglu:
                    oracle.swiglu_f64(y)
            n += 1
            if time.perf_counter() - t >= budget_s:
                break
        sec = (time.perf_counter() - t) / n
        return sec, f"{n} full steps (all {w.M} rows, every GEMM) in {sec * n:.1f} s", nthreads
    # row sample: rows spread over the groups, time scaled by M / rows
    k = max(nthreads, int(budget_s / max(sum(per_row), 1e-9)))
    k = min(k, w.M)
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(w.M, size=k, replace=False))
    t = time.perf_counter()
    oracle.moe_align(prob.topk_np, w.E)
    for d in prob.gemms:
        oracle.grouped_gemm_f64(d["x_np"], d["packed_np"], d["absmax_np"], sizes, experts, rows=rows)
    el = time.perf_counter() - t
    sec = t_align + (el - t_align) * w.M / k
    return sec, (f"{k} of {w.M} rows per GEMM (seeded sample) in {el:.1f} s; full-step time "
                 f"extrapolated x{w.M / k:.1f} by rows"), nthreads


def metric_value(prob, sec_per_step, n_ranks=1):
    if prob.prefill:
        return prob.step_flops * n_ranks / sec_per_step / 1e12, "TFLOP/s"
    return prob.step_bytes * n_ranks / sec_per_step / 1e9, "GB/s"


def run_reference(args, rank, world):
    """The oracle (plain C, fp64) on the host cores, on our arm's workload,
    metric and config. Host-only: the product library is never imported."""
    if rank != 0:
        return None
    prob = HostProblem(args.workload, seed=0)
    budget = max(3.0, min(60.0, 2.0 * (args.steps + args.warmup)))
    sec, sample, threads = oracle_step_sample(prob, budget)
    val, unit = metric_value(prob, sec)
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": prob.describe(),
        "cpu_baseline": {"value": val, "unit": unit, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "timing": "the oracle on the host cores (no GPU, no graph)",
    }
    line["config"]["parallelism"] = "single GPU" if world <= 1 else f"replicas x{world}"
    return line


def side_record(res, pk, cpu_budget, glue):
    """What one non-headline workload contributes to the line: its step
    throughput, per-call times, per-GEMM roofline, clocks and oracle baseline."""
    prob = res["prob"]
    sec = res["ms"] / 1e3 / res["steps"]
    val, unit = metric_value(prob, sec)
    rec = {"value": val, "unit": unit, "ms_per_step": res["ms"] / res["steps"],
           "steps": res["steps"], "warmup": res["warmup"], "config": prob.describe(),
           "kernels": kernels_entry(prob, res["kern_ms"]),
           "roofline": {d["g"].name: roofline(prob, d, res["kern_ms"][1 + i], pk)
                        for i, d in enumerate(prob.gemms)},
           "step_kernels": res["step_kernels"], "clocks": res["clocks"]}
    if glue is not None:
        rec["glue"] = glue
    if cpu_budget > 0:
        sec_cpu, sample, threads = oracle_step_sample(prob, cpu_budget)
        v, u = metric_value(prob, sec_cpu)
        rec["cpu_baseline"] = {"value": v, "unit": u, "cores": threads, "kind": "oracle",
                               "sample": sample}
    return rec


# --------------------------------------------------------------------- main
HEADLINE = "mixtral_8x22b"
SIDE_STEPS = {"tiny": 5000, "olmoe": 5000, "qwen3_30b_a3b": 2000, "gpt_oss_120b": 300,
              "mixtral_8x22b": 50}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE, choices=list(synth.WORKLOADS),
                    help="the headline workload (default: the largest single-GPU config)")
    ap.add_argument("--only", action="store_true",
                    help="time only the headline workload (skip the other configs)")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of CPU time for the headline's oracle baseline sample")
    ap.add_argument("--side-cpu-budget", type=float, default=5.0,
                    help="seconds of CPU time for each other config's oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = DEFAULT_STEPS[args.workload]
    if args.warmup is None:
        args.warmup = max(3, args.steps // 20)
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        # rank 0 alone times the oracle; the other ranks exit without work
        line = run_reference(args, rank, world)
        if rank == 0:
            print(json.dumps(line))
        return

    if world > 1:
        timeout = __import__("datetime").timedelta(seconds=120)
        if torch.cuda.is_available():
            torch.cuda.set_device(local_rank)
            torch.distributed.init_process_group(
                "nccl", device_id=torch.device("cuda", local_rank), timeout=timeout)
        else:   # host-only runs (tests): gloo
            torch.distributed.init_process_group("gloo", timeout=timeout)

    import grouped_nf4_w4a16_b200 as gnf4
    gnf4.load_library()    # fails loudly if the CUDA library is missing
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    drv = _cuda_driver()
    pk = peaks()

    res = run_ours(args.workload, args.steps, args.warmup, world, dev, stream, drv)
    prob = res["prob"]
    ms, kern_ms = res["ms"], res["kern_ms"]
    sec = ms / 1e3 / args.steps
    val, unit = metric_value(prob, sec, world)
    # the glue entry points after the step's numbers: an error there is
    # reported in the line instead of costing them
    try:
        glue = time_glue(prob, stream)
    except Exception as exc:   # noqa: BLE001
        glue = {"error": f"{type(exc).__name__}: {exc}"}

    roofs = {d["g"].name: roofline(prob, d, kern_ms[1 + i], pk) for i, d in enumerate(prob.gemms)}
    e2e_ms, h2d, d2h, e2e_steps = res["e2e"]
    e2e_val, _ = metric_value(prob, e2e_ms / 1e3, world)
    kpl = len(res["step_kernels"]) if res["step_kernels"] is not None else None
    line = {
        "metric": METRIC, "value": val, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": prob.describe(),
        # the dominant kernel: the gate_up GEMM launch (the larger of the two)
        "roofline": roofs[prob.gemms[0]["g"].name],
        "roofline_per_gemm": roofs,
        "kernels": kernels_entry(prob, kern_ms),
        "glue": glue,
        "e2e": {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "how": ("eager C-ABI calls; every step copies its inputs in from pinned host memory and "
                        "its results out to pinned host memory, pipelined: copies in and out on two "
                        "copy streams overlap the previous / next step's compute over two sets of "
                        "device buffers")},
        "gpu_launches": kpl * args.steps if kpl is not None else None,
        "step_kernels": res["step_kernels"],
        "timing": ("each step is one CUDA graph of the C-ABI calls (moe_align, then each GEMM); "
                   "per-call times from event nodes in a copy of the graph"),
        "clocks": res["clocks"],
    }
    line["config"]["parallelism"] = f"replicas x{world}" if world > 1 else "single GPU"
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sec_cpu, sample, threads = oracle_step_sample(prob, args.cpu_budget)
        v, u = metric_value(prob, sec_cpu)
        line["cpu_baseline"] = {"value": v, "unit": u, "cores": threads, "kind": "oracle",
                                "sample": sample}
    prob.free()
    del res, prob
    torch.cuda.empty_cache()

    # the other configurations, one GPU only: each one's step throughput,
    # per-GEMM roofline and oracle baseline under "configs"
    if world == 1 and not args.only:
        others = {}
        for name in synth.WORKLOADS:
            if name == args.workload:
                continue
            try:
                r = run_ours(name, SIDE_STEPS[name], max(3, SIDE_STEPS[name] // 20), 1, dev,
                             stream, drv, with_e2e=False)
                try:
                    g = time_glue(r["prob"], stream)
                except Exception as exc:   # noqa: BLE001
                    g = {"error": f"{type(exc).__name__}: {exc}"}
                others[name] = side_record(r, pk, 0.0 if args.no_cpu_baseline
                                           else args.side_cpu_budget, g)
                r["prob"].free()
                del r
                torch.cuda.empty_cache()
            except Exception as exc:   # noqa: BLE001
                others[name] = {"error": f"{type(exc).__name__}: {exc}"}
        line["configs"] = others
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
