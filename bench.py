#!/usr/bin/env python
"""Benchmark of the NVFP4 weight-only MoE branch on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode64|decode1|dense1|aff4_64|prefill4096|block64|
                                block4096|stack30|quantize]

A step is one pass of the whole hot path -- route, permute, gate_up + GELU,
down, combine -- over one batch of synthetic tokens (the default workload:
one MoE layer of the Gemma-4-26B-A4B shapes, T=64 decode tokens; the default
run also times the T=4096 prefill workload on the same layer and reports it
under "prefill", the metric's tensor-core half).  Inputs are
resident in HBM before the timed region; L2 is flushed (256 MiB write)
between timed steps, outside the timed events.  Each rank runs its own replica
(the branch is per-token independent; no collective on the data path);
`value` is the tokens all ranks processed / max-over-ranks time.

--impl reference times the CPU oracle (numpy, fp64) on a bounded sample of
the same workload on the host cores; with N>1 only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s; decode HBM GB/s vs ~8 TB/s; prefill TFLOP/s vs bf16 peak"
GU_EXPERT_BYTES = 1408 * 1408 + 1408 * 176 + 4        # packed + scales + global
DN_EXPERT_BYTES = 2816 * 352 + 2816 * 44 + 4
EXPERT_BYTES = GU_EXPERT_BYTES + DN_EXPERT_BYTES        # 3,345,416
AFF4_GU_BYTES = 1408 * 1408 + 1408 * 88 * 4             # codes + fp16 scales and biases per 32
AFF4_EXPERT_BYTES = AFF4_GU_BYTES + 2816 * 352 + 2816 * 22 * 4   # 3,717,120
ROUTER_BYTES = 128 * 2816 * 2 + 2816 * 2 + 128 * 2       # 726,784 (bf16 proj, scale, pes)
FLUSH_BYTES = 256 << 20

# DRAM read + write per launch of each workload's dominant kernel, as taken
# by an ncu capture, with the SHA-256 of the kernel's source files at capture
# time; a figure whose sources have changed since is reported as null.
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def source_digest(paths) -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in sorted(paths):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(rel.encode() + b"\0" + f.read())
    return h.hexdigest()


def captured_traffic(workload: str):
    """(bytes per launch, kernel) of the workload's dominant kernel from the
    capture file, or (None, None) if absent or taken on other sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)[workload]
        if rec["sources_sha256"] != source_digest(rec["sources"]):
            return None, rec.get("kernel")
        return float(rec["dram_bytes_per_launch"]), rec.get("kernel")
    except Exception:
        return None, None

WORKLOADS = {
    "decode64": {"T": 64, "layers": 1, "zipf": False,
                 "desc": "one MoE layer (H=2816, E=128, top-8, I=704, NVFP4 experts), decode T=64"},
    "decode1": {"T": 1, "layers": 1, "zipf": False, "desc": "one MoE layer, decode T=1"},
    "prefill4096": {"T": 4096, "layers": 1, "zipf": True,
                    "desc": "one MoE layer, prefill T=4096, Zipf(1.1)-skewed router bias"},
    "aff4_64": {"T": 64, "layers": 1, "zipf": False, "aff4": True,
                "desc": "one MoE layer with aff4 experts (u4, fp16 scale+bias per 32), decode T=64"},
    "w4a4_64": {"T": 64, "layers": 1, "zipf": False, "w4a4": True,
                "desc": "one MoE layer in the W4A4 form (NVFP4 activations, block-scaled FP4 tensor cores), decode T=64"},
    "w4a4_4096": {"T": 4096, "layers": 1, "zipf": True, "w4a4": True,
                  "desc": "one MoE layer in the W4A4 form, prefill T=4096, Zipf(1.1)-skewed router bias"},
    "dense1": {"T": 1, "layers": 1, "zipf": False, "dense": True,
               "desc": "one MoE layer, decode T=1, dense over-read: all 128 experts per token (ablation)"},
    "block64": {"T": 64, "layers": 1, "zipf": False, "block": True,
                "desc": "full MoE block (dense MLP 2112 || NVFP4 experts, norms, layer scalar), decode T=64"},
    "block4096": {"T": 4096, "layers": 1, "zipf": True, "block": True,
                  "desc": "full MoE block, prefill T=4096, Zipf(1.1)-skewed router bias"},
    "stack30": {"T": 8, "layers": 30, "zipf": False,
                "desc": "30 independently seeded MoE layers chained x+=moe(rmsnorm(x)), T=8"},
    "quantize": {"T": 0, "layers": 0, "zipf": False,
                 "desc": "nvfp4_quantize of bf16 [128,1408,2816] N(0,0.02) with 0.5% x20 outliers"},
}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            p = [c.strip() for c in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax.append(float(p[2]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def physical_gpu_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


# --------------------------------------------------------------- oracle
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


class OracleSample:
    """The oracle on a bounded sample of the workload: inputs are generated
    once; each run() times one oracle pass over the sample."""

    def __init__(self, workload: str, wl: dict, tokens: int):
        import moe_inputs as gen
        self.workload, self.tokens = workload, tokens
        if workload == "quantize":
            self.w = gen.make_quant_weights(4, 1, 1408, 2816)
            self.what = "oracle quantize of 1 of the 128 expert tensors [1408,2816]"
            return
        self.ex = gen.make_experts(0 if wl["layers"] == 1 else 100)
        if wl.get("aff4"):
            from oracle import aff4 as A
            self.ex = A.Aff4Experts(*gen.make_aff4_experts(9))
        self.rt = gen.make_router(1, bias=gen.zipf_bias(7) if wl["zipf"] else None)
        self.x = gen.make_x(10_000, max(wl["T"], tokens))[:tokens]
        self.block = None
        if wl.get("block"):
            from oracle import block as B
            b = gen.make_block(200)
            self.block = B.BlockParams(self.ex, self.rt, b.dense_gate, b.dense_up, b.dense_down, b.pre_ff_norm,
                                       b.post_ff_norm_1, b.pre_ff_norm_2, b.post_ff_norm_2, b.post_ff_norm,
                                       b.layer_scalar)
        self.w4a4 = bool(wl.get("w4a4"))
        self.what = (f"oracle fp64 forward of {tokens} of the workload's tokens through one "
                     + ("full block" if self.block else ("W4A4 layer" if self.w4a4 else "layer")))

    def run(self):
        """Returns (value, unit, seconds)."""
        from oracle import moe as M
        from oracle import quantize as Q
        t0 = time.perf_counter()
        if self.workload == "quantize":
            Q.quantize(self.w)
            dt = time.perf_counter() - t0
            nbytes = self.w.nbytes + self.w.nbytes // 4 + self.w.nbytes // 16 + 4
            return nbytes / dt / 1e9, "GB/s", dt
        if self.block is not None:
            from oracle import block as B
            B.forward(self.x, self.block)
        elif self.w4a4:
            import moe_inputs as gen
            from oracle import w4a4 as W
            W.forward(self.x, self.ex, self.rt, gen.W4A4_GX, gen.W4A4_GH)
        else:
            M.forward(self.x, self.ex, self.rt)
        dt = time.perf_counter() - t0
        return self.tokens / dt, "tokens/s", dt


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    tokens = 4 if args.workload in ("prefill4096", "w4a4_4096") else 2
    sample = OracleSample(args.workload, wl, tokens)
    what = sample.what
    for _ in range(min(args.warmup, 1)):
        sample.run()
    vals, secs = [], []
    for _ in range(args.steps):
        v, unit, dt = sample.run()
        vals.append(v)
        secs.append(dt)
    total = sum(secs)
    value = (tokens * args.steps / total) if unit == "tokens/s" else statistics.mean(vals)
    if args.workload == "stack30":
        value /= 30.0   # a stack step runs 30 layers
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": args.workload, "desc": wl["desc"]},
        "cpu_baseline": {"value": value, "unit": unit, "cores": blas_threads(), "kind": "oracle",
                         "sample": what + f", {args.steps} steps"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------ replica aggregation
def max_over_ranks(value: float, world: int, device) -> float:
    """The largest `value` over all ranks (every rank gets it): step times
    are reported as the slowest replica's."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput: the units all replicas processed over `steps`
    steps, divided by the (slowest replica's) time."""
    return world * units_per_rank * steps / (total_ms / 1e3)


def replica_x_seed(rank: int, n_pool: int, i: int) -> int:
    """Seed of input i of a replica's pool: disjoint pools across ranks."""
    return 10_000 + rank * n_pool + i


# ----------------------------------------------------------------- ours
class _Ctx:
    """Per-process state shared by the measured workloads."""

    def __init__(self, rank, world, local_rank):
        import torch
        self.rank, self.world, self.local_rank = rank, world, local_rank
        self.dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(self.dev)
        self.flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=self.dev)
        self.hbm_peak, self.tc_peak, self.tc_peak_sus, self.peak_kind = measured_peaks()
        self._experts = {}

    def experts(self, seed):
        """Device copy of a layer's experts with their packed code tiles (made
        once at load, like the quantisation itself; the decode kernels stream
        them as whole blocks), shared by workloads on the same seed."""
        import moe_inputs as gen
        import nvfp4_weight_only_router_b200 as lib
        if seed not in self._experts:
            ex = gen.make_experts(seed)
            self._experts[seed] = lib.Experts.from_host(ex, self.dev).packed()
            del ex
        return self._experts[seed]


def _bf(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def measure(ctx, workload, args, cpu_baseline=True):
    """Time one workload: W warm-up steps (and at least --min-warmup-s of
    load), then exactly K timed steps between L2 flushes, CUDA events on the
    launching stream, max over ranks.  Returns the JSON-line fields."""
    import ctypes
    import torch
    import torch.distributed as dist
    import moe_inputs as gen
    import nvfp4_weight_only_router_b200 as lib
    from nvfp4_weight_only_router_b200 import capi

    wl = WORKLOADS[workload]
    rank, world, dev = ctx.rank, ctx.world, ctx.dev
    T = wl["T"]
    n_pool = 64
    extra = {}
    events = [torch.cuda.Event(enable_timing=True) for _ in range(6)]

    if workload == "quantize":
        w = gen.make_quant_weights(4, 128, 1408, 2816)
        w_pin = _bf(w).pin_memory()  # host copy of the weights for the end-to-end pass
        wd = w_pin.to(dev)
        del w
        q = torch.empty((128, 1408, 1408), dtype=torch.uint8, device=dev)
        s = torch.empty((128, 1408, 176), dtype=torch.uint8, device=dev)
        g = torch.empty((128,), dtype=torch.float32, device=dev)
        q_pin = torch.empty(q.shape, dtype=torch.uint8).pin_memory()
        s_pin = torch.empty(s.shape, dtype=torch.uint8).pin_memory()
        g_pin = torch.empty(g.shape, dtype=torch.float32).pin_memory()
        ws_bytes = capi.nvfp4_quantize_workspace_bytes(128, 1408, 2816)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

        def step(i):
            capi.check(capi.nvfp4_quantize(wd.data_ptr(), 128, 1408, 2816, q.data_ptr(), s.data_ptr(),
                                           g.data_ptr(), ws.data_ptr(), ws_bytes,
                                           torch.cuda.current_stream().cuda_stream))

        def prepare(i):
            pass
        algo_bytes = wd.numel() * 2 + q.numel() + s.numel() + 128 * 4
        kernels_per_step = 1  # the single-pass kernel (the clearing of its counters is a memset)
    else:
        layers = []
        seeds = [0] if wl["layers"] == 1 else gen.layer_seed_plan(wl["layers"])
        for sd in seeds:
            rt = gen.make_router(1 if wl["layers"] == 1 else 1000 + sd,
                                 bias=gen.zipf_bias(7) if wl["zipf"] else None)
            if wl.get("block"):
                parts = lib.DenseParts.from_host(gen.make_block(200), dev)
                layers.append(lib.MoeBlock(ctx.experts(sd), lib.Router.from_host(rt, dev), parts, max_tokens=T))
            elif wl.get("w4a4"):
                layers.append(lib.W4A4Layer(ctx.experts(sd), lib.Router.from_host(rt, dev), gen.W4A4_GX, gen.W4A4_GH,
                                            max_tokens=T))
            elif wl.get("aff4"):
                layers.append(lib.Aff4Layer(lib.Aff4Experts.from_host(gen.make_aff4_experts(9), dev),
                                            lib.Router.from_host(rt, dev), max_tokens=T))
            else:
                layers.append(lib.MoeLayer(ctx.experts(sd), lib.Router.from_host(rt, dev), max_tokens=T))
        xs_host = np.stack([gen.make_x(replica_x_seed(rank, n_pool, i), T) for i in range(n_pool)])
        x_pool = _bf(xs_host).to(dev)
        x_pin = _bf(xs_host).pin_memory()
        xs = torch.empty((T, 2816), dtype=torch.bfloat16, device=dev)
        y = torch.empty_like(xs)
        y_pin = torch.empty((T, 2816), dtype=torch.bfloat16).pin_memory()
        res = torch.empty((T, 2816), dtype=torch.float32, device=dev)
        xn = torch.empty_like(xs)

        def fwd_layer(layer, xin, yout, profiled):
            st = torch.cuda.current_stream().cuda_stream
            if wl.get("dense"):
                layer.forward_dense_into(xin, yout)
            elif wl.get("block") or wl.get("aff4"):
                layer.forward_into(xin, yout)
            elif profiled and wl.get("w4a4"):
                arr = (ctypes.c_void_p * 6)(*[ctypes.c_void_p(e.cuda_event) for e in events])
                capi.check(capi.moe_w4a4_forward_profiled(
                    xin.data_ptr(), T, ctypes.byref(layer._xs), ctypes.byref(layer._rs), yout.data_ptr(),
                    layer.workspace.data_ptr(), layer.workspace.numel(), st, arr))
            elif profiled:
                arr = (ctypes.c_void_p * 6)(*[ctypes.c_void_p(e.cuda_event) for e in events])
                capi.check(capi.moe_nvfp4_forward_profiled(
                    xin.data_ptr(), T, ctypes.byref(layer._xs), ctypes.byref(layer._rs), yout.data_ptr(),
                    layer.workspace.data_ptr(), layer.workspace.numel(), st, arr))
            else:
                layer.forward_into(xin, yout)

        def step_body(profiled):
            if len(layers) == 1:
                fwd_layer(layers[0], xs, y, profiled)
            else:
                res.copy_(xs.float())
                lib.residual_rmsnorm(res, None, xn)
                for li, layer in enumerate(layers):
                    fwd_layer(layer, xn, y, profiled and li == 0)
                    lib.residual_rmsnorm(res, y, xn)

        for e in events:   # events must have been recorded once before capture use
            e.record()
        torch.cuda.synchronize()
        # capture one step into a CUDA graph (fixed pointers; inputs rotate into xs)
        xs.copy_(x_pool[0])
        step_body(True)
        torch.cuda.synchronize()
        # two graphs of the same step: a plain one for the timed steps, and one
        # with event-record nodes between the phases for the phase breakdown
        # (event nodes cost launch gaps, so they stay out of the headline time)
        graph_prof = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_prof):
            step_body(True)
        torch.cuda.synchronize()
        step_body(False)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step_body(False)
        torch.cuda.synchronize()

        def step(i):
            graph.replay()

        def step_prof(i):
            graph_prof.replay()

        def prepare(i):
            xs.copy_(x_pool[i % n_pool])

        # per layer: route (with the permutation when T*8 <= 1024, else two
        # permutation kernels), gather, gate_up, down, combine; plus the
        # chain's rmsnorm kernels
        per_layer = 5 if T * 8 <= 1024 else 7
        if wl.get("dense"):
            per_layer = 6  # route, dense permutation, gather, gate_up, down, combine
        if wl.get("block"):
            # prenorm, the routed branch without its combine, dense gate_up,
            # GELU, dense down, the block's final kernel
            per_layer = (4 if T * 8 <= 1024 else 6) + 5
        kernels_per_step = per_layer * len(layers) + (len(layers) + 1 if len(layers) > 1 else 0)

    # -------- warm-up (at least W steps and at least --min-warmup-s, so the clock sampler sees load)
    sampler = ClockSampler(physical_gpu_index(ctx.local_rank))
    t_end = time.perf_counter() + args.min_warmup_s
    i = 0
    while i < args.warmup or time.perf_counter() < t_end:
        prepare(i)
        step(i)
        i += 1
    torch.cuda.synchronize()

    # -------- timed steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step_ms, phase_ms, act_counts = [], [], []
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for k in range(args.steps):
        ctx.flush.zero_()
        prepare(k)
        start.record()
        step(k)
        end.record()
        torch.cuda.synchronize()
        step_ms.append(start.elapsed_time(end))
        if workload != "quantize" and not (wl.get("block") or wl.get("aff4")):
            act_counts.append(int((layers[0].views(T)["counts"] > 0).sum().item()))
        elif wl.get("block") or wl.get("aff4"):
            act_counts.append(int(torch.unique(layers[0].ids(T)).numel()))
    torch.cuda.synchronize()
    # phase breakdown (and the dominant kernel's duration for the roofline):
    # the same K steps again, each replaying the graph whose event-record
    # nodes sit between the phases, on the launching stream
    prof_ms = []
    if workload != "quantize":
        for k in range(args.steps):
            if wl.get("dense") or wl.get("block") or wl.get("aff4"):
                break  # these variants record no phase events
            ctx.flush.zero_()
            prepare(k)
            start.record()
            step_prof(k)
            end.record()
            torch.cuda.synchronize()
            prof_ms.append(start.elapsed_time(end))
            phase_ms.append([events[j].elapsed_time(events[j + 1]) for j in range(5)])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()

    total_ms = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms / args.steps

    # -------- e2e through the public API with host buffers
    if workload == "quantize":
        # the weights come from pinned host memory and the codes, scales and
        # global scales go back to it, every step
        e_ms = []
        for k in range(args.steps):
            ctx.flush.zero_()
            torch.cuda.synchronize()
            start.record()
            wd.copy_(w_pin, non_blocking=True)
            step(k)
            q_pin.copy_(q, non_blocking=True)
            s_pin.copy_(s, non_blocking=True)
            g_pin.copy_(g, non_blocking=True)
            end.record()
            end.synchronize()
            e_ms.append(start.elapsed_time(end))
        e_tot = max_over_ranks(sum(e_ms), world, dev)
        e2e = {"value": job_rate(algo_bytes, world, args.steps, e_tot) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": wd.numel() * 2,
               "d2h_bytes_per_step": q.numel() + s.numel() + g.numel() * 4}
    else:
        e_ms = []
        for k in range(args.steps):
            ctx.flush.zero_()
            torch.cuda.synchronize()
            start.record()
            xs.copy_(x_pin[k % n_pool], non_blocking=True)
            step_body(False)
            y_pin.copy_(y, non_blocking=True)
            end.record()
            end.synchronize()
            e_ms.append(start.elapsed_time(end))
        e_tot = max_over_ranks(sum(e_ms), world, dev)
        e2e = {"value": job_rate(T, world, args.steps, e_tot), "unit": "tokens/s",
               "h2d_bytes_per_step": T * 2816 * 2, "d2h_bytes_per_step": T * 2816 * 2}

    # -------- roofline of the dominant kernel
    traffic, traffic_kernel = captured_traffic(workload)
    if workload == "quantize":
        value = job_rate(algo_bytes, world, args.steps, total_ms) / 1e9
        unit = "GB/s"
        roof = {"bound": "hbm", "kernel": "quantize_fused_kernel (single pass: amax + encode)",
                "achieved": algo_bytes / (ms_per_step / 1e3) / 1e9, "peak": ctx.hbm_peak, "unit": "GB/s",
                "traffic": traffic, "peak_kind": ctx.peak_kind, "algorithmic_per_launch": float(algo_bytes)}
        roof["frac"] = roof["achieved"] / roof["peak"]
        dtype = "u8"
    else:
        value = job_rate(T, world, args.steps, total_ms)
        unit = "tokens/s"
        ph = np.array(phase_ms) if phase_ms else np.full((1, 5), np.nan)  # route, permute, gate_up, down, combine
        n_act = np.array(act_counts, np.float64)
        if wl.get("dense"):
            n_act = np.full_like(n_act, 128.0)  # every expert is read
        S = T * 8
        gu_bytes = n_act * GU_EXPERT_BYTES + T * 2816 * 2 + S * 704 * 2
        gu_flops = 2.0 * S * 1408 * 2816
        gu_ms = ph[:, 2]
        dense_bytes = 3 * 2816 * 2112 * 2
        dense_flops = 2.0 * T * 3 * 2816 * 2112
        if wl.get("w4a4") and T >= 1024:
            # FP4 x FP4 on the tensor cores: the burst bf16 peak x the nominal fp4 / bf16 ratio (9 / 2.25)
            ach = gu_flops / (gu_ms.mean() / 1e3) / 1e12
            roof = {"bound": "tensor", "kernel": "gate_up W4A4 grouped GEMM + GELU + hidden quantisation (tcgen05 mxf4nvf4)",
                    "achieved": ach, "peak": ctx.tc_peak * 4.0, "unit": "TFLOP/s", "traffic": traffic,
                    "peak_kind": ctx.peak_kind + " burst bf16 x 4 (nominal fp4/bf16)",
                    "algorithmic_per_launch": gu_flops}
        elif wl.get("w4a4"):
            # weights + the slots' activation codes and scales in, hidden codes and scales out
            w4_bytes = n_act * GU_EXPERT_BYTES + S * (1408 + 176) + S * (352 + 44)
            ach = w4_bytes.sum() / (gu_ms.sum() / 1e3) / 1e9
            roof = {"bound": "hbm", "kernel": "gate_up W4A4 grouped GEMM + GELU + hidden quantisation (tcgen05 mxf4nvf4)",
                    "achieved": ach, "peak": ctx.hbm_peak, "unit": "GB/s", "traffic": traffic,
                    "peak_kind": ctx.peak_kind, "algorithmic_per_launch": float(w4_bytes.mean())}
        elif wl.get("block") and T >= 1024:
            flops = 2.0 * S * (1408 * 2816 + 2816 * 704) + dense_flops
            ach = flops / (ms_per_step / 1e3) / 1e12
            roof = {"bound": "tensor", "kernel": "whole block step (experts + dense MLP, no phase split)",
                    "achieved": ach, "peak": ctx.tc_peak, "unit": "TFLOP/s", "traffic": traffic,
                    "peak_kind": ctx.peak_kind + " burst bf16", "algorithmic_per_launch": flops}
        elif wl.get("block"):
            nbytes = (n_act * EXPERT_BYTES + ROUTER_BYTES + dense_bytes + 2 * T * 2816 * 2).mean()
            ach = nbytes / (ms_per_step / 1e3) / 1e9
            roof = {"bound": "hbm", "kernel": "whole block step (experts + dense MLP, no phase split)",
                    "achieved": ach, "peak": ctx.hbm_peak, "unit": "GB/s", "traffic": traffic,
                    "peak_kind": ctx.peak_kind, "algorithmic_per_launch": float(nbytes)}
        elif T >= 1024:
            # a sub-millisecond kernel timed between L2 flushes: the burst peak
            ach = gu_flops / (gu_ms.mean() / 1e3) / 1e12
            roof = {"bound": "tensor", "kernel": "gate_up grouped GEMM + GELU (tcgen05)", "achieved": ach,
                    "peak": ctx.tc_peak, "unit": "TFLOP/s", "traffic": traffic,
                    "peak_kind": ctx.peak_kind + " burst bf16", "algorithmic_per_launch": gu_flops}
        elif wl.get("aff4"):
            nbytes = (n_act * AFF4_EXPERT_BYTES + ROUTER_BYTES + 2 * T * 2816 * 2).mean()
            ach = nbytes / (ms_per_step / 1e3) / 1e9
            roof = {"bound": "hbm", "kernel": "whole aff4 step (no phase split)", "achieved": ach,
                    "peak": ctx.hbm_peak, "unit": "GB/s", "traffic": traffic, "peak_kind": ctx.peak_kind,
                    "algorithmic_per_launch": float(nbytes)}
        elif wl.get("dense"):
            # no phase split: the whole step's algorithmic bytes (all 128 experts)
            ach = (n_act * EXPERT_BYTES + ROUTER_BYTES + 2 * T * 2816 * 2).mean() / (ms_per_step / 1e3) / 1e9
            roof = {"bound": "hbm", "kernel": "whole dense over-read step (all experts)", "achieved": ach,
                    "peak": ctx.hbm_peak, "unit": "GB/s", "traffic": traffic, "peak_kind": ctx.peak_kind,
                    "algorithmic_per_launch": float((n_act * EXPERT_BYTES).mean())}
        else:
            ach = gu_bytes.sum() / (gu_ms.sum() / 1e3) / 1e9
            roof = {"bound": "hbm", "kernel": "gate_up grouped GEMV + GELU", "achieved": ach,
                    "peak": ctx.hbm_peak, "unit": "GB/s", "traffic": traffic,
                    "peak_kind": ctx.peak_kind,
                    "algorithmic_per_launch": float(gu_bytes.mean())}
        roof["frac"] = roof["achieved"] / roof["peak"]
        step_bytes = n_act * EXPERT_BYTES + ROUTER_BYTES + 2 * T * 2816 * 2
        extra = {
            "phase_ms_mean": None if (wl.get("dense") or wl.get("block") or wl.get("aff4")) else dict(zip(["route", "permute", "gate_up", "down", "combine"],
                                                                 [float(v) for v in ph.mean(0)])),
            "ms_per_step_with_phase_events": float(np.mean(prof_ms)) if prof_ms else None,
            "active_experts_mean": float(n_act.mean()),
            # whole-step algorithmic bytes (active experts + router + x + y) per second
            "step_hbm_gbs": float(step_bytes.mean() * wl["layers"] / (ms_per_step / 1e3) / 1e9),
            "layer_tflops": float(2.0 * S * (1408 * 2816 + 2816 * 704) * wl["layers"] / (ms_per_step / 1e3) / 1e12),
        }
        dtype = "e2m1xe2m1" if wl.get("w4a4") else "f16xe2m1"
    if traffic_kernel:
        roof["traffic_kernel"] = traffic_kernel

    cpu = None
    if rank == 0 and cpu_baseline:
        tokens = 4 if workload in ("prefill4096", "w4a4_4096") else 2
        sample = OracleSample(workload, wl, tokens)
        v, u, dt = sample.run()
        what = sample.what
        if workload == "stack30":
            v /= 30.0
            what += " (value per 30-layer step)"
        cpu = {"value": v, "unit": u, "cores": blas_threads(), "kind": "oracle",
               "sample": what + f" ({dt:.1f} s)"}

    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "config": {"workload": workload, "desc": wl["desc"], "T": T,
                   "l2": "256 MiB flush write between timed steps",
                   "graph": workload != "quantize", "parallelism": f"replicas x{world}",
                   "weights": None if workload == "quantize" or wl.get("aff4") else "NVFP4 codes + packed 16 KB code tiles"},
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": kernels_per_step * args.steps, "clocks": clocks,
    }
    line.update(extra)
    if workload != "quantize":
        del graph, graph_prof
    return line


def run_ours(args, rank, world, local_rank):
    import torch.distributed as dist
    from nvfp4_weight_only_router_b200 import build as bld

    if rank == 0 or world == 1:
        bld.build()
    if world > 1:
        dist.barrier()
    ctx = _Ctx(rank, world, local_rank)
    line = measure(ctx, args.workload, args, cpu_baseline=not args.no_cpu_baseline)
    if args.workload == "decode64" and not args.no_prefill:
        # the metric's other half: the prefill workload on the same experts, in
        # the same invocation (its own warm-up, timed steps and clock record)
        p = measure(ctx, "prefill4096", args, cpu_baseline=False)
        line["prefill"] = {k: p[k] for k in ("value", "unit", "ms_per_step", "roofline", "clocks", "e2e",
                                             "gpu_launches", "phase_ms_mean", "layer_tflops")}
        line["prefill"]["config"] = p["config"]
    if args.workload == "decode64" and not args.no_w4a4:
        # the W4A4 form of the same layer (NVFP4 activations on the FP4 tensor
        # cores), decode and prefill, in the same invocation
        for key, w in (("w4a4_decode", "w4a4_64"), ("w4a4_prefill", "w4a4_4096")):
            q = measure(ctx, w, args, cpu_baseline=False)
            line[key] = {k: q[k] for k in ("value", "unit", "ms_per_step", "roofline", "clocks", "e2e",
                                           "gpu_launches", "phase_ms_mean", "dtype")}
            line[key]["config"] = q["config"]
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode64", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-w4a4", action="store_true",
                    help="decode64: skip the W4A4 decode and prefill lines")
    ap.add_argument("--no-prefill", action="store_true",
                    help="decode64 only: skip the prefill4096 half of the metric")
    ap.add_argument("--min-warmup-s", type=float, default=1.0,
                    help="keep warming up for at least this long (the clock sampler needs load)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
