#!/usr/bin/env python
"""Benchmark of the streaming int4 MoE stack on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Default workload ``decode_b1_l40``: one decode step = one token of one stream through all
40 MoE layers (d=2048, 256 experts + 1 shared, I=512, top-4, int4 affine g64, LoRA r=16
on the shared expert, 33 linear prerouter heads whose predictions are the next step's
routing).  Weights and inputs are seeded synthetic draws (``synth``); the expert weights
(18.1 GB) exceed L2, and each step reads ~406 MB of them.

Prints one JSON line.  ``value`` is tokens/s with inputs resident in HBM; ``e2e`` is the
same metric through the C ABI with the step's inputs copied from pinned host memory and
its outputs copied back inside the timed region.  With N > 1 (torchrun) every rank runs
an independent replica (the path has no exchange step) and ``value`` is the sum over
ranks divided by the slowest rank's time.

``--impl reference`` times the CPU oracle (float64 numpy) on bounded samples of the same
workload on the host cores.
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

import synth  # noqa: E402

METRIC = "MoE-stack decode tokens/s on 1 B200; achieved HBM GB/s vs ~8 TB/s peak"

# DRAM bytes (read + write) per launch of the dominant kernel from an ncu capture, valid only
# while the kernel's code is the one captured: sha256 prefix of its source files (the
# kernel's file and the headers it includes) with comments removed and white space
# collapsed, so that comment edits keep the numbers; see profiles/.
KERNEL_TRAFFIC = {
    "decode_b1_l40": (("int4_expert_streaming_prerouter_b200/csrc/e0_decode.cuh",
                       "int4_expert_streaming_prerouter_b200/csrc/e0_kernels.cuh",
                       "int4_expert_streaming_prerouter_b200/csrc/e0_device.cuh"), "2e9b3dd381860134", 409.9e6,
                      "4-layer capture (40.99 MB DRAM per launch for 40.67 MB algorithmic) scaled by algorithmic "
                      "bytes to the 40-layer launch"),
    "prefill_t4096_l40": (("int4_expert_streaming_prerouter_b200/csrc/e0_prefill.cuh",
                           "int4_expert_streaming_prerouter_b200/csrc/e0_kernels.cuh",
                           "int4_expert_streaming_prerouter_b200/csrc/e0_device.cuh"), "d088c3d2737d7eff", 343.6e6,
                          "k_moe_gemm_tc DRAM bytes per launch on one full-width layer (T=4096): gate/up 465.8 MB, "
                          "down 221.4 MB, mean of the two"),
}


def code_digest(paths):
    """sha256 of C/C++/CUDA sources (one path or several, in order) with // and /* */
    comments removed (string and character literals kept) and every run of white space
    collapsed to one blank."""
    import hashlib
    if isinstance(paths, str):
        paths = (paths,)
    src = "\n".join(open(p, encoding="utf-8").read() for p in paths)
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return hashlib.sha256(" ".join("".join(out).split()).encode()).hexdigest()


def kernel_traffic(workload):
    ent = KERNEL_TRAFFIC.get(workload)
    if not ent:
        return None, None
    paths, digest, nbytes, how = ent
    h = code_digest([os.path.join(ROOT, p) for p in paths])
    return (nbytes, how) if h.startswith(digest) else (None, "kernel changed since the capture")
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(PEAKS_FALLBACK, source="fallback")


# ---------------------------------------------------------------------------------------
# algorithmic bytes of one decode step (what the kernels must read at least once)
# ---------------------------------------------------------------------------------------
def step_bytes(dims, idx, B):
    """idx [L, B, k] routing of the step.  Returns (expert bytes, all bytes)."""
    blob = synth.blob_bytes(dims.d, dims.I)
    d, E, I, r = dims.d, dims.E, dims.I, dims.r
    expert = other = 0
    heads = set(dims.head_layers)
    for n in range(dims.L):
        u = len(set(idx[n].reshape(-1).tolist()))
        expert += (u + 1) * blob                            # routed uniques + shared expert
        predicted = n > 0 and (n - 1) in heads
        other += (B * dims.k * d * 2) if predicted else E * d * 2   # router rows
        other += E * d * 2 if n in heads else 0                     # head
        other += (2 * r * d + 2 * I * r + r * I + d * r) * 2        # LoRA
        other += d * 2                                               # gamma
        other += B * d * 2 * 2                                       # h in, y out (bf16)
    return expert, expert + other


# ---------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event reasons of one GPU during a timed region.  Two sources run
    side by side: NVML read every 5 ms from a thread (enough samples for short regions),
    and `nvidia-smi -lms 100`; the summary uses the NVML samples when there are any.  Only
    reads; nothing is set.  `nvml` may be a stand-in module (tests)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, gpu_index: int, nvml=None, use_smi: bool = True):
        self.gpu = gpu_index
        self.proc = None
        self.use_smi = use_smi
        self.nvml = nvml
        self.samples = []            # NVML: (sm MHz, reason bits)
        self.max_mhz = None
        self.thread = None
        self.stop = None
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"e0_clocks_rank{gpu_index}.csv")
        self.uuid = None
        try:
            import torch
            u = str(torch.cuda.get_device_properties(gpu_index).uuid)
            self.uuid = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            pass

    def _nvml_start(self):
        import threading
        nv = self.nvml
        if nv is None:
            import pynvml as nv
        nv.nvmlInit()
        h = nv.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid else nv.nvmlDeviceGetHandleByIndex(self.gpu)
        reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        self.stop = threading.Event()

        def loop():
            while not self.stop.is_set():
                try:
                    self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)), int(reasons(h))))
                except Exception:
                    return
                self.stop.wait(0.005)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def __enter__(self):
        try:
            self._nvml_start()
        except Exception:
            self.thread = None
        if self.use_smi:
            try:
                os.makedirs(os.path.dirname(self.path), exist_ok=True)
                self.f = open(self.path, "w")
                sel = [f"--id={self.uuid}"] if self.uuid else []
                self.proc = subprocess.Popen(["nvidia-smi"] + sel + [f"--query-gpu={self.Q}",
                                              "--format=csv,noheader,nounits", "-lms", "100"],
                                             stdout=self.f, stderr=subprocess.DEVNULL)
            except Exception:
                self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.samples:
            sm = [m for m, _ in self.samples]
            reasons = sorted({name for _, bits in self.samples for name, bit in self.REASONS if bits & bit})
            return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                    "samples": len(sm), "source": "nvml, 5 ms"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) >= 9 and p[1].replace(".", "").isdigit():
                rows.append(p)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        reasons = set()
        for r in rows:
            for name, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                               r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": sorted(reasons),
                "samples": len(rows), "source": "nvidia-smi, 100 ms"}


# ---------------------------------------------------------------------------------------
# distributed plumbing (replicas only)
# ---------------------------------------------------------------------------------------
def dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        # NCCL between GPUs; gloo where there is no GPU (the plumbing's CPU tests)
        dist.init_process_group("nccl" if torch.cuda.is_available() else "gloo",
                                timeout=datetime.timedelta(seconds=300))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce(v: float, op):
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(v: float, ws: int) -> float:
    if ws == 1:
        return v
    import torch.distributed as dist
    return _reduce(v, dist.ReduceOp.MAX)


def sum_over_ranks(v: float, ws: int) -> float:
    if ws == 1:
        return v
    import torch.distributed as dist
    return _reduce(v, dist.ReduceOp.SUM)


# ---------------------------------------------------------------------------------------
# CPU oracle timing (baseline / reference arm)
# ---------------------------------------------------------------------------------------
def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def oracle_decode_sample(dims, seed, n_layers: int, step: int = 0):
    """Time the oracle on one token of one stream through the first `n_layers` layers
    (own-router routing, as at step 0).  Returns seconds."""
    import oracle as O
    hs = synth.hidden(seed, step, dims.L, 1, dims.d)
    t0 = time.perf_counter()
    for n in range(n_layers):
        dense = synth.layer_dense(seed, n, dims)
        out = O.moe_layer(hs[n], dense, lambda e, n=n: synth.expert_blob(seed, n, e, dims),
                          synth.shared_blob(seed, n, dims), dims)
        if n in dims.head_layers:
            O.prerouter_head(out["x"][0], dense, dims)
    return time.perf_counter() - t0


def cpu_baseline(dims, seed, budget_s=20.0):
    """The oracle as it stands on a bounded sample: whole layers of one token, as many as
    fit the budget; tokens/s is extrapolated to the 40-layer stack."""
    t1 = oracle_decode_sample(dims, seed, 1)
    n = int(max(1, min(dims.L, budget_s / max(t1, 1e-3))))
    t = oracle_decode_sample(dims, seed, n)
    per_token = t * dims.L / n
    return {"value": 1.0 / per_token, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"1 token (B=1) through {n} of {dims.L} layers, own-router routing; "
                      f"time scaled x{dims.L / n:.2f} to the full stack (incl. weight generation per layer)"}


def run_reference(args, dims, seed, ws, rank):
    if rank != 0:
        return
    per_step_layers = None
    times = []
    for i in range(args.warmup + args.steps):
        if per_step_layers is None:
            t1 = oracle_decode_sample(dims, seed, 1)
            # keep the whole run within ~3 minutes
            per_step_layers = int(max(1, min(dims.L, 180.0 / max(1, args.warmup + args.steps) / max(t1, 1e-3))))
        t = oracle_decode_sample(dims, seed, per_step_layers, step=i)
        if i >= args.warmup:
            times.append(t * dims.L / per_step_layers)
    per_token = sum(times) / len(times)
    v = 1.0 / per_token
    sample = (f"each step: 1 token (B=1) through {per_step_layers} of {dims.L} layers, "
              f"time scaled to the full stack")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_token * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "layers": dims.L, "batch": 1, "d": dims.d, "experts": dims.E},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ---------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------
def run_decode(args, dims, seed, B, ws, rank, local):
    import torch
    import int4_expert_streaming_prerouter_b200 as e0
    from synth.device import layer_tensors, bf16_tensor

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    t0 = time.time()
    ctx = e0.Context(dims.d, dims.E, dims.I, dims.k, dims.r, dims.L, max(B, 1))
    lys, hds = [], []
    for n in range(dims.L):
        ly, hd = layer_tensors(seed, n, dims, dev)
        lys.append(ly)
        hds.append(hd)
    ctx.register_model(lys, hds)
    ctx.debug_decode_mode(args.decode_mode)
    if args.decode_flat is not None:
        ctx.debug_decode_flat(args.decode_flat)
    setup_s = time.time() - t0
    steps, warm = args.steps, args.warmup
    total = steps + warm
    # every step has its own generated inputs, resident before the timed region
    h_all = torch.stack([bf16_tensor(synth.hidden(seed, t, dims.L, B, dims.d), dev) for t in range(total)])
    y = torch.empty((dims.L, B, dims.d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    for t in range(warm):
        ctx.stack_decode(h_all[t], t, y_out=y)
    ctx.sync_status()
    launches0 = ctx.stats()["kernel_launches"]
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    routes = []
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for t in range(warm, total):
            ctx.stack_decode(h_all[t], t, y_out=y)
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    ctx.sync_status()
    ms = ev0.elapsed_time(ev1)
    launches = ctx.stats()["kernel_launches"] - launches0
    idx, _ = ctx.get_routing(B)
    exp_b, all_b = step_bytes(dims, idx, B)
    ms_max = max_over_ranks(ms, ws)
    tokens = sum_over_ranks(B * steps, ws)
    value = tokens / (ms_max / 1e3)

    # end-to-end through the C ABI with host buffers (e0_moe_stack_decode_host): every
    # step's input copied in from pinned host memory and its output copied back, the
    # library overlapping those copies with the neighbouring steps' kernels
    h_host = torch.empty((steps, dims.L, B, dims.d), dtype=torch.bfloat16, pin_memory=True)
    h_host.copy_(h_all[warm:].cpu())
    y_host = torch.empty((steps, dims.L, B, dims.d), dtype=torch.bfloat16, pin_memory=True)
    torch.cuda.synchronize()
    nxt = total          # continue the same decode sequence
    barrier(ws)
    e0_, e1_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0_.record(stream)
    for t in range(steps):
        ctx.stack_decode_host(h_host[t], nxt + t, y_host[t])
    ctx.host_io_wait()
    e1_.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    e2e_ms = max_over_ranks(e0_.elapsed_time(e1_), ws)
    e2e_value = tokens / (e2e_ms / 1e3)

    pk = peaks()
    step_ms = ms / steps
    achieved = exp_b / (step_ms / 1e3) / 1e9
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": steps, "warmup": warm,
        "ms_per_step": ms_max / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 weights, fp32 accumulate", "data": "synthetic (seeded random weights and inputs of the model's shapes)",
        "config": {"workload": args.workload, "layers": dims.L, "batch": B, "d": dims.d, "experts": dims.E,
                   "d_ff": dims.I, "top_k": dims.k, "lora_rank": dims.r, "heads": len(dims.head_layers),
                   "parallelism": f"replicas x{ws}", "l2": "inputs larger than L2 (18.1 GB of expert weights)"},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": int(h_host[0].numel() * 2),
                "d2h_bytes_per_step": int(y_host[0].numel() * 2)},
        "gpu_launches": int(launches),
        "hbm": {"expert_bytes_per_step": exp_b, "all_bytes_per_step": all_b,
                "expert_GBps": achieved, "all_GBps": all_b / (step_ms / 1e3) / 1e9,
                "frac_of_measured": achieved / pk["hbm_gbs"], "frac_of_8TBps": achieved / 8000.0},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "traffic": kernel_traffic(args.workload)[0],
                     "traffic_note": kernel_traffic(args.workload)[1],
                     "kernel": ("k_decode (one launch = one decode step, CUDA events on its stream); "
                                "achieved counts int4 expert bytes only" if B == 1 else
                                "per-layer kernels of one decode step; achieved counts int4 expert bytes"),
                     "peak_source": pk["source"] + " copy bandwidth (burst)"},
        "clocks": clk.summary(),
        "setup_s": setup_s,
    }
    return out, ctx


def run_prefill(args, dims, seed, ws, rank, local):
    """One step = one prefill chunk of T tokens through all layers."""
    import torch
    import int4_expert_streaming_prerouter_b200 as e0
    from synth.device import layer_tensors, bf16_tensor

    T = synth.WORKLOADS[args.workload]["tokens"]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    t0 = time.time()
    ctx = e0.Context(dims.d, dims.E, dims.I, dims.k, dims.r, dims.L, T)
    lys, hds = zip(*[layer_tensors(seed, n, dims, dev) for n in range(dims.L)])
    ctx.register_model(list(lys), list(hds))
    h = torch.stack([bf16_tensor(synth.prefill_hidden(seed, n, T, dims.d), dev) for n in range(dims.L)])
    setup_s = time.time() - t0
    y = torch.empty_like(h)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        ctx.prefill_stack(h, y_out=y)
    ctx.sync_status()
    st0 = ctx.stats()
    ctx.debug_time_gemm(True)   # event pairs around every expert-GEMM launch, on its stream
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            ctx.prefill_stack(h, y_out=y)
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    ctx.sync_status()
    ctx.debug_time_gemm(False)
    ms = max_over_ranks(ev0.elapsed_time(ev1), ws)
    st1 = ctx.stats()
    launches = st1["kernel_launches"] - st0["kernel_launches"]
    gemm_n = st1["gemm_timed"] - st0["gemm_timed"]
    gemm_ms = max_over_ranks(st1["gemm_ms"] - st0["gemm_ms"], ws)
    tokens = sum_over_ranks(T * args.steps, ws)
    # algorithmic expert FLOPs: every token through k routed + the shared expert, gate and
    # up (2 d I each) and down (2 I d), per layer
    flops = dims.L * T * (dims.k + 1) * (2 * dims.d * 2 * dims.I + 2 * dims.I * dims.d)
    pk = peaks()
    step_s = ms / args.steps / 1e3
    # the dominant kernel: the expert GEMMs' FLOPs over their own measured launch time
    achieved = flops * args.steps / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else flops / step_s / 1e12
    traffic, traffic_how = kernel_traffic(args.workload)
    # end to end: the chunk's inputs from pinned host memory, its outputs back
    h_host = h.cpu().pin_memory()
    y_host = torch.empty_like(h_host).pin_memory()
    e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_a.record(stream)
    for _ in range(args.steps):
        h.copy_(h_host, non_blocking=True)
        ctx.prefill_stack(h, y_out=y)
        y_host.copy_(y, non_blocking=True)
    e_b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_a.elapsed_time(e_b), ws)
    out = {
        "metric": "MoE-stack prefill tokens/s on 1 B200 (4096-token chunk, 40 layers)", "value": tokens / (ms / 1e3),
        "unit": "tokens/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 weights as exact bf16 tensor-core operands (128+q), bf16 activations, fp32 accumulate",
        "data": "synthetic (seeded)",
        "config": {"workload": args.workload, "layers": dims.L, "tokens": T, "d": dims.d, "experts": dims.E,
                   "d_ff": dims.I, "top_k": dims.k, "parallelism": f"replicas x{ws}",
                   "l2": "inputs larger than L2 (18.1 GB of expert weights)"},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h.numel() * 2),
                "d2h_bytes_per_step": int(y.numel() * 2)},
        "gpu_launches": int(launches),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / pk["bf16_tflops"], "traffic": traffic,
                     "kernel": f"k_moe_gemm_tc ({gemm_n} launches timed, {gemm_ms / max(gemm_n, 1):.3f} ms mean; "
                               f"expert FLOPs of the chunk / their summed time; "
                               f"{100 * gemm_ms / max(ms, 1e-9):.0f}% of the step)",
                     "traffic_note": traffic_how, "peak_source": pk["source"]},
        "clocks": clk.summary(), "setup_s": setup_s,
    }
    return out, ctx


def h2d_probe_gbs(dev, nbytes=1 << 28):
    """Pinned host -> device copy bandwidth (GB/s), measured once in this run."""
    import torch
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    for _ in range(2):
        dst.copy_(src, non_blocking=True)
    torch.cuda.synchronize()
    e0_, e1_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0_.record()
    for _ in range(4):
        dst.copy_(src, non_blocking=True)
    e1_.record()
    torch.cuda.synchronize()
    return 4 * nbytes / (e0_.elapsed_time(e1_) / 1e3) / 1e9


def run_stream(args, dims, seed, ws, rank, local):
    """Streaming tier: experts in pinned host memory, staged into a 2 x k slot pool."""
    import torch
    import int4_expert_streaming_prerouter_b200 as e0
    from synth.device import layer_tensors, bf16_tensor, pinned_expert_store

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    t0 = time.time()
    ctx = e0.Context(dims.d, dims.E, dims.I, dims.k, dims.r, dims.L, 1)
    lys, hds = zip(*[layer_tensors(seed, n, dims, dev, resident=False) for n in range(dims.L)])
    ctx.register_model(list(lys), list(hds))
    store = pinned_expert_store(seed, dims)
    ctx.stream_register(store, pool_layers=2, slots_per_layer=dims.k)
    setup_s = time.time() - t0
    total = args.warmup + args.steps
    h_all = torch.stack([bf16_tensor(synth.hidden(seed, t, dims.L, 1, dims.d), dev) for t in range(total)])
    y = torch.empty((dims.L, 1, dims.d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    for t in range(args.warmup):
        ctx.stack_decode(h_all[t], t, y_out=y, streaming=True)
    ctx.sync_status()
    s0 = ctx.stats()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for t in range(args.warmup, total):
            ctx.stack_decode(h_all[t], t, y_out=y, streaming=True)
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    ctx.sync_status()
    s1 = ctx.stats()
    ms = max_over_ranks(ev0.elapsed_time(ev1), ws)
    tokens = sum_over_ranks(args.steps, ws)
    d = {k: s1[k] - s0[k] for k in s1}
    link = h2d_probe_gbs(dev)
    bytes_per_token = d["staged_bytes"] / args.steps
    wall_s = ms / 1e3
    out = {
        "metric": "MoE-stack streaming decode tokens/s on 1 B200 (experts in pinned host memory)",
        "value": tokens / wall_s, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 weights, fp32 accumulate", "data": "synthetic (seeded)",
        "config": {"workload": args.workload, "layers": dims.L, "batch": 1, "pool": f"2 layers x {dims.k} slots",
                   "host_store_GB": round(store.numel() / 1e9, 2), "parallelism": f"replicas x{ws}"},
        "gpu_launches": int(d["kernel_launches"]),
        "streaming": {"host_link_bytes_per_token": bytes_per_token, "h2d_probe_GBps": link,
                      "link_GBps": bytes_per_token * tokens / wall_s / 1e9,
                      "link_frac": bytes_per_token * tokens / wall_s / 1e9 / link,
                      "stage_ms_per_token": d["stage_ms"] / args.steps,
                      "exposed_wait_ms_per_token": d["exposed_wait_ms"] / args.steps,
                      "hidden_frac_of_staging": 1.0 - d["exposed_wait_ms"] / max(d["stage_ms"], 1e-9),
                      "link_busy_frac_of_wall": d["stage_ms"] / max(ms, 1e-9),
                      "prefetched_experts": int(d["prefetched_experts"]),
                      "ondemand_experts": int(d["ondemand_experts"]), "dropped": int(d["dropped"]),
                      "hbm_pool_MB": 2 * dims.k * synth.blob_bytes(dims.d, dims.I) / 1e6},
        "roofline": {"bound": "host link", "achieved": bytes_per_token * tokens / wall_s / 1e9, "peak": link,
                     "unit": "GB/s", "frac": bytes_per_token * tokens / wall_s / 1e9 / link, "traffic": None,
                     "kernel": "staging copies (copy engine)", "peak_source": "pinned H2D probe in this run"},
        "clocks": clk.summary(), "setup_s": setup_s,
    }
    return out, ctx


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1024)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--workload", default="decode_b1_l40")
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-mode", type=int, default=0, help="0 default, 1 one-launch, 2 graph, 3 eager")
    ap.add_argument("--decode-flat", type=int, default=None,
                    help="one-launch kernel on unchained steps: 1 flat schedule (default), 0 layers in order")
    args = ap.parse_args()
    wl = synth.WORKLOADS[args.workload]
    dims, seed = wl["dims"], wl["seed"]
    ws, rank, local = dist_init() if args.impl == "ours" else (int(os.environ.get("WORLD_SIZE", "1")),
                                                                int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        run_reference(args, dims, seed, ws, rank)
        return
    if args.workload.startswith("stream"):
        out, ctx = run_stream(args, dims, seed, ws, rank, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
        ctx.close()
        return
    if "tokens" in wl:
        out, ctx = run_prefill(args, dims, seed, ws, rank, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
        ctx.close()
        return
    B = args.batch or (wl["batch"] if isinstance(wl.get("batch"), int) else 8)
    out, ctx = run_decode(args, dims, seed, B, ws, rank, local)
    if rank == 0:
        if not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(dims, seed)
        print(json.dumps(out), flush=True)
    ctx.close()
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
