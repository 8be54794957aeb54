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
                       "int4_expert_streaming_prerouter_b200/csrc/e0_device.cuh"), "5c7d623b5c947fb3", 408.6e6,
                      "4-layer capture (40.86 MB DRAM per launch for 40.67 MB algorithmic) scaled by algorithmic "
                      "bytes to the 40-layer launch"),
    "prefill_t4096_l40": (("int4_expert_streaming_prerouter_b200/csrc/e0_prefill.cuh",
                           "int4_expert_streaming_prerouter_b200/csrc/e0_kernels.cuh",
                           "int4_expert_streaming_prerouter_b200/csrc/e0_device.cuh"), "19732f9b31a4e06e", 318.6e6,
                          "k_moe_gemm_tc DRAM bytes per launch on one full-width layer (T=4096): gate/up 422.3 MB, "
                          "down 214.9 MB, mean of the two"),
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
def step_bytes(dims, idx, B, parts=False):
    """idx [L, B, k] routing of the step.  Returns (expert bytes, all bytes), or with
    parts=True a dict: gate/up and down expert bytes, bf16 rows (routers, heads, LoRA A)
    and the rest."""
    blob = synth.blob_bytes(dims.d, dims.I)
    d, E, I, r = dims.d, dims.E, dims.I, dims.r
    gu_bytes = 2 * (I * d // 2 + 2 * I * (d // 64) * 2)          # gate + up of one expert
    dn_bytes = blob - gu_bytes
    gu = dn = rows = rest = 0
    heads = set(dims.head_layers)
    for n in range(dims.L):
        u = len(set(idx[n].reshape(-1).tolist())) + 1             # routed uniques + shared expert
        gu += u * gu_bytes
        dn += u * dn_bytes
        predicted = n > 0 and (n - 1) in heads
        rows += min(B * dims.k, E) * d * 2 if predicted else E * d * 2     # router rows
        rows += E * dims.head_in * 2 if n in heads else 0                   # head
        rows += 2 * r * d * 2                                                # LoRA A_g, A_u
        rest += (2 * I * r + r * I + d * r) * 2                              # LoRA B_g, B_u, A_d, B_d
        rest += d * 2 + B * d * 2 * 2                                        # gamma, h in, y out
    if parts:
        return {"gate_up": gu, "down": dn, "rows": rows, "rest": rest}
    return gu + dn, gu + dn + rows + rest


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


def _oracle_layer_inputs(dims, seed, n, h_bits):
    """The weights the oracle needs for one layer on the given tokens, drawn before any
    timing: the dense weights, the shared expert and the routed experts that the layer's own
    router selects (a cheap routing pass over the same inputs)."""
    import oracle as O
    dense = synth.layer_dense(seed, n, dims)
    x = O.rmsnorm(O.bf16_to_f64(h_bits), dense["norm_w"], dims.eps)
    lg = O.router_logits(dense["router_w"], x)
    used = sorted({int(e) for t in range(lg.shape[0]) for e in O.topk(lg[t], dims.k)})
    blobs = {e: synth.expert_blob(seed, n, e, dims) for e in used}
    return dense, blobs, synth.shared_blob(seed, n, dims)


def oracle_decode_sample(dims, seed, n_layers: int, step: int = 0):
    """Time the oracle on one token of one stream through the first `n_layers` layers
    (own-router routing, as at step 0), the layer's head included.  Weights are drawn
    before the clock starts.  Returns seconds."""
    import oracle as O
    hs = synth.hidden(seed, step, dims.L, 1, dims.d)
    pre = [_oracle_layer_inputs(dims, seed, n, hs[n]) for n in range(n_layers)]
    t0 = time.perf_counter()
    for n in range(n_layers):
        dense, blobs, shared = pre[n]
        out = O.moe_layer(hs[n], dense, blobs.__getitem__, shared, dims)
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
            "sample": f"1 token (B=1) through {n} of {dims.L} layers, own-router routing, heads included; "
                      f"time scaled x{dims.L / n:.2f} to the full stack; weights drawn before timing"}


def cpu_baseline_tokens(dims, seed, hs_layer, layer: int, scale_layers: int, what: str):
    """The oracle on the given tokens of one layer (own-router routing), weights drawn
    before timing; tokens/s of the whole stack = tokens / (time x scale_layers)."""
    import oracle as O
    dense, blobs, shared = _oracle_layer_inputs(dims, seed, layer, hs_layer)
    t0 = time.perf_counter()
    O.moe_layer(hs_layer, dense, blobs.__getitem__, shared, dims)
    t = time.perf_counter() - t0
    T = hs_layer.shape[0]
    return {"value": T / (t * scale_layers), "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{what}: {T} tokens through layer {layer} (own-router routing), time scaled "
                      f"x{scale_layers} to the {dims.L}-layer stack; weights drawn before timing"}


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
              f"time scaled to the full stack; weights drawn before timing")
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
def _free_gpu():
    import gc
    import torch
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _load_model(dims, seed, dev, resident=True):
    import int4_expert_streaming_prerouter_b200 as e0
    from synth.device import layer_tensors
    lys, hds = [], []
    for n in range(dims.L):
        ly, hd = layer_tensors(seed, n, dims, dev, resident=resident)
        lys.append(ly)
        hds.append(hd)
    return lys, hds


def _context(dims, lys, hds, max_tokens):
    import int4_expert_streaming_prerouter_b200 as e0
    ctx = e0.Context(dims.d, dims.E, dims.I, dims.k, dims.r, dims.L, max_tokens,
                     head_hidden=dims.head_hidden, head_onehot=dims.head_onehot)
    ctx.register_model(lys, hds)
    return ctx


def _timed_steps(ctx, h_all, t0, n, y, ws, local, chained=False, streaming=False):
    """n decode steps t0..t0+n-1 bracketed by CUDA events on the launching stream, barrier
    and synchronisation on both sides; returns (ms, clocks, kernel launches, routing of the
    last step)."""
    import torch
    stream = torch.cuda.current_stream()
    ctx.sync_status()
    l0 = ctx.stats()["kernel_launches"]
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for t in range(t0, t0 + n):
            ctx.stack_decode(h_all[t % len(h_all)], t, y_out=y, chained=chained, streaming=streaming)
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    ctx.sync_status()
    return ev0.elapsed_time(ev1), clk.summary(), ctx.stats()["kernel_launches"] - l0


def _hbm_roofline(bytes_per_step, ms_per_step, pk, kernel, traffic=None, note=None):
    ach = bytes_per_step / (ms_per_step / 1e3) / 1e9
    out = {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": ach / pk["hbm_gbs"],
           "traffic": traffic, "kernel": kernel, "peak_source": pk["source"] + " copy bandwidth (burst)"}
    if note:
        out["traffic_note"] = note
    return out


PHASE_NAMES = ("k_ph_norm", "k_ph_rows", "k_ph_route", "k_ph_gateup", "k_ph_tdsum", "k_ph_down")


def phase_breakdown(ctx, h_all, t0, n, y, parts, pk):
    """Per-kernel CUDA-event times of the phased decode kernels (launched one after another
    for this pass only) and each streaming kernel's achieved HBM bandwidth on its
    algorithmic bytes."""
    ms0, n0 = ctx.debug_phase_times()
    ctx.debug_phase_timing(True)
    for t in range(t0, t0 + n):
        ctx.stack_decode(h_all[t % len(h_all)], t, y_out=y)
    ctx.debug_phase_timing(False)
    ms1, n1 = ctx.debug_phase_times()
    steps = n1 - n0
    if steps <= 0:
        return None
    per = [(b - a) / steps for a, b in zip(ms0, ms1)]
    nbytes = {"k_ph_rows": parts["rows"], "k_ph_gateup": parts["gate_up"], "k_ph_down": parts["down"]}
    out = {"ms_per_step_serialised": sum(per), "steps": steps, "kernels": {}}
    for name, m in zip(PHASE_NAMES, per):
        ent = {"ms": m}
        if name in nbytes:
            ent["algorithmic_bytes"] = nbytes[name]
            ent["GBps"] = nbytes[name] / (m / 1e3) / 1e9
            ent["frac"] = ent["GBps"] / pk["hbm_gbs"]
        out["kernels"][name] = ent
    return out


def run_decode(args, dims, seed, B, ws, rank, local, extras):
    import torch
    import int4_expert_streaming_prerouter_b200 as e0
    from synth.device import bf16_tensor

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    t0 = time.time()
    lys, hds = _load_model(dims, seed, dev)
    ctx = _context(dims, lys, hds, max(B, 1))
    ctx.debug_decode_mode(args.decode_mode)
    if args.decode_flat is not None:
        ctx.debug_decode_flat(args.decode_flat)
    setup_s = time.time() - t0
    steps, warm = args.steps, args.warmup
    total = steps + warm
    # every step has its own generated inputs, resident before the timed region
    h_all = torch.stack([bf16_tensor(synth.hidden(seed, t, dims.L, B, dims.d), dev) for t in range(total + 16)])
    y = torch.empty((dims.L, B, dims.d), dtype=torch.bfloat16, device=dev)
    for t in range(warm):
        ctx.stack_decode(h_all[t], t, y_out=y)
    ms, clocks, launches = _timed_steps(ctx, h_all, warm, steps, y, ws, local)
    idx, _ = ctx.get_routing(B)
    parts = step_bytes(dims, idx, B, parts=True)
    exp_b = parts["gate_up"] + parts["down"]
    all_b = exp_b + parts["rows"] + parts["rest"]
    ms_max = max_over_ranks(ms, ws)
    tokens = sum_over_ranks(B * steps, ws)
    value = tokens / (ms_max / 1e3)

    # end to end through the C ABI with host buffers (e0_moe_stack_decode_host): every
    # step's input copied in from pinned host memory and its output copied back, the
    # library overlapping those copies with the neighbouring steps' kernels
    stream = torch.cuda.current_stream(dev)
    h_host = torch.empty((steps, dims.L, B, dims.d), dtype=torch.bfloat16, pin_memory=True)
    h_host.copy_(h_all[warm:total].cpu())
    y_host = torch.empty((steps, dims.L, B, dims.d), dtype=torch.bfloat16, pin_memory=True)
    nxt = total          # continue the same decode sequence
    # one untimed call first: the library allocates its host-I/O staging buffers on first use
    ctx.stack_decode_host(h_host[0], nxt, y_host[0])
    ctx.host_io_wait()
    torch.cuda.synchronize()
    nxt += 1
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
    nxt += steps

    pk = peaks()
    step_ms = ms / steps
    phased = args.decode_mode == 4 or (args.decode_mode == 0 and 2 <= B <= 64)
    traffic, how = kernel_traffic("decode_b1_l40_phased" if phased else args.workload) if B == 1 else (None, None)
    kernel = ("decode step = six phased kernels (norm, bf16 rows, routing, gate/up, sums, down) launched "
              "with programmatic dependent launch; CUDA events around the timed steps on their stream; "
              "achieved counts int4 expert bytes only" if phased else
              "k_decode (one launch = one decode step, CUDA events on its stream); achieved counts int4 "
              "expert bytes only" if B == 1 else
              "per-layer kernels of one decode step; achieved counts int4 expert bytes")
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
                "expert_GBps": exp_b / (step_ms / 1e3) / 1e9, "all_GBps": all_b / (step_ms / 1e3) / 1e9,
                "frac_of_measured": exp_b / (step_ms / 1e3) / 1e9 / pk["hbm_gbs"],
                "frac_of_8TBps": exp_b / (step_ms / 1e3) / 1e9 / 8000.0},
        "roofline": _hbm_roofline(exp_b, step_ms, pk, kernel, traffic, how),
        "clocks": clocks,
        "setup_s": setup_s,
    }
    if phased:
        pb = phase_breakdown(ctx, h_all, nxt, 8, y, parts, pk)
        nxt += 8
        if pb:
            out["phased_kernels"] = pb
    if extras:
        # the one-launch persistent kernel on the same unchained steps, and the chained step
        # (layer N's input is bf16(h_N + y_{N-1}): layers in order, as a real decoder runs)
        n_x = min(steps, 64)
        sub = {}
        for name, mode, chained in (("one_launch_unchained", 1, False), ("chained_in_order", 0, True)):
            ctx.debug_decode_mode(mode)
            for t in range(2):
                ctx.stack_decode(h_all[t], t, y_out=y, chained=chained)
            ms_x, clk_x, l_x = _timed_steps(ctx, h_all, 2, n_x, y, ws, local, chained=chained)
            ms_x = max_over_ranks(ms_x, ws)
            sub[name] = {"value": sum_over_ranks(B * n_x, ws) / (ms_x / 1e3), "unit": "tokens/s",
                         "ms_per_step": ms_x / n_x, "steps": n_x, "gpu_launches": int(l_x),
                         "roofline": _hbm_roofline(exp_b, ms_x / n_x, pk,
                                                   "k_decode (one cooperative launch per step; in layer order "
                                                   "when chained)"),
                         "clocks": clk_x}
        ctx.debug_decode_mode(args.decode_mode)
        out["decode_variants"] = sub
    return out, ctx


def run_prefill(args, dims, seed, ws, rank, local, T=4096):
    """One step = one prefill chunk of T tokens through all layers."""
    import torch
    from synth.device import bf16_tensor

    T = synth.WORKLOADS[args.workload].get("tokens", T)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    t0 = time.time()
    lys, hds = _load_model(dims, seed, dev)
    ctx = _context(dims, lys, hds, T)
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
    traffic, traffic_how = kernel_traffic("prefill_t4096_l40")
    # end to end through the C ABI with host buffers (e0_moe_prefill_stack_host): every
    # layer's input copied in from pinned host memory and its output copied back, the
    # copies of one layer beside the kernels of its neighbours
    h_host = h.cpu().pin_memory()
    y_host = torch.empty_like(h_host).pin_memory()
    ctx.prefill_stack_host(h_host, y_host)   # untimed: the staging buffers are allocated on first use
    ctx.host_io_wait()
    torch.cuda.synchronize()
    e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_a.record(stream)
    for _ in range(args.steps):
        ctx.prefill_stack_host(h_host, y_host)
    ctx.host_io_wait()
    e_b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_a.elapsed_time(e_b), ws)
    out = {
        "metric": "MoE-stack prefill tokens/s on 1 B200 (4096-token chunk, 40 layers)", "value": tokens / (ms / 1e3),
        "unit": "tokens/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 weights as two exact fp16 tensor-core operands (s(q&14), s(q&1)), bf16-valued fp16 activations, fp32 accumulate",
        "data": "synthetic (seeded)",
        "config": {"workload": "prefill_t4096_l40", "layers": dims.L, "tokens": T, "d": dims.d, "experts": dims.E,
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
    return out, ctx, h


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


def _stream_case(ctx, dims, h_all, warm, steps, ws, local, link, B=1, e2e=False):
    """Streamed decode steps; tok/s, host-link bytes per token and the staging accounting."""
    import torch
    y = torch.empty((dims.L, B, dims.d), dtype=torch.bfloat16, device=h_all.device)
    for t in range(warm):
        ctx.stack_decode(h_all[t], t, y_out=y, streaming=True)
    ctx.sync_status()
    s0 = ctx.stats()
    ms, clocks, _ = _timed_steps(ctx, h_all, warm, steps, y, ws, local, streaming=True)
    s1 = ctx.stats()
    idx_rec = None
    d = {k: s1[k] - s0[k] for k in s1}
    ms = max_over_ranks(ms, ws)
    tokens = sum_over_ranks(B * steps, ws)
    wall_s = ms / 1e3
    bpt = d["staged_bytes"] / (B * steps)
    link_gbps = d["staged_bytes"] / wall_s / 1e9
    req = d["staged_experts"] + d["hit_experts"]
    out = {"value": tokens / wall_s, "unit": "tokens/s", "ms_per_step": ms / steps, "steps": steps, "batch": B,
           "host_link_bytes_per_token": bpt, "link_GBps": link_gbps, "link_frac": link_gbps / link,
           "stage_ms_per_step": d["stage_ms"] / steps, "exposed_wait_ms_per_step": d["exposed_wait_ms"] / steps,
           "hidden_frac_of_staging": 1.0 - d["exposed_wait_ms"] / max(d["stage_ms"], 1e-9),
           "link_busy_frac_of_wall": d["stage_ms"] / max(ms, 1e-9),
           "copied_experts": int(d["staged_experts"]), "hit_experts": int(d["hit_experts"]),
           "hit_rate": d["hit_experts"] / max(req, 1),
           "prefetched_experts": int(d["prefetched_experts"]), "ondemand_experts": int(d["ondemand_experts"]),
           "dropped": int(d["dropped"]), "gpu_launches": int(d["kernel_launches"]), "clocks": clocks,
           "roofline": {"bound": "host link", "achieved": link_gbps, "peak": link, "unit": "GB/s",
                        "frac": link_gbps / link, "traffic": None, "kernel": "staging copies (copy engine)",
                        "peak_source": "pinned H2D probe in this run"}}
    if e2e:
        # the step's input from pinned host memory and its output back, through the C ABI
        h_host = h_all[warm:warm + steps].cpu().pin_memory()
        y_host = torch.empty((steps, dims.L, B, dims.d), dtype=torch.bfloat16, pin_memory=True)
        t_base = warm + steps
        stream = torch.cuda.current_stream()
        ctx.stack_decode_host(h_host[0], t_base, y_host[0], streaming=True)   # untimed: allocates
        ctx.host_io_wait()
        t_base += 1
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for t in range(steps):
            ctx.stack_decode_host(h_host[t], t_base + t, y_host[t], streaming=True)
        ctx.host_io_wait()
        b.record(stream)
        torch.cuda.synchronize()
        ms_e = max_over_ranks(a.elapsed_time(b), ws)
        out["e2e"] = {"value": tokens / (ms_e / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h_host[0].numel() * 2),
                      "d2h_bytes_per_step": int(y_host[0].numel() * 2)}
    return out


def run_stream(args, dims, seed, ws, rank, local, variants=True):
    """Streaming tier: experts in pinned host memory, staged into HBM slot sets.  The
    workload's configuration (two shared 4-slot sets, prefetch from the predictions) is the
    headline; with `variants`, the same model also runs the fully reactive mode, persistent
    sticky sets, and both on inputs shaped to the multi-stream routing statistics (next-token
    reuse ~0.44), plus a least-recently-used HBM cache at batch 8."""
    import torch
    import int4_expert_streaming_prerouter_b200 as e0
    from synth.device import bf16_tensor, pinned_expert_store

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    t0 = time.time()
    lys, hds = _load_model(dims, seed, dev, resident=False)
    store = pinned_expert_store(seed, dims)
    setup_s = time.time() - t0
    link = h2d_probe_gbs(dev)
    warm, steps = args.warmup, args.steps
    total = warm + 2 * steps + 2
    h_all = torch.stack([bf16_tensor(synth.hidden(seed, t, dims.L, 1, dims.d), dev) for t in range(total)])

    def case(pool_layers, slots, reactive, h, B=1, e2e=False):
        ctx = _context(dims, lys, hds, B)
        ctx.stream_register(store, pool_layers=pool_layers, slots_per_layer=slots)
        ctx.stream_mode(reactive)
        r = _stream_case(ctx, dims, h, warm, steps, ws, local, link, B=B, e2e=e2e)
        idx, _ = ctx.get_routing(B)
        ctx.close()
        r["config"] = {"pool_sets": pool_layers, "slots_per_set": slots, "mode": "reactive" if reactive else "prefetch",
                       "hbm_pool_MB": pool_layers * slots * synth.blob_bytes(dims.d, dims.I) / 1e6}
        return r

    head = case(2, dims.k, False, h_all, e2e=True)
    out = {
        "metric": "MoE-stack streaming decode tokens/s on 1 B200 (experts in pinned host memory)",
        "value": head["value"], "unit": "tokens/s", "n_gpus": ws, "steps": steps, "warmup": warm,
        "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 weights, fp32 accumulate", "data": "synthetic (seeded)",
        "config": {"workload": "stream_b1_l40", "layers": dims.L, "batch": 1, "pool": f"2 layers x {dims.k} slots",
                   "host_store_GB": round(store.numel() / 1e9, 2), "parallelism": f"replicas x{ws}"},
        "gpu_launches": head["gpu_launches"], "e2e": head["e2e"],
        "streaming": {k: v for k, v in head.items() if k not in ("roofline", "clocks", "e2e", "gpu_launches")},
        "roofline": head["roofline"], "clocks": head["clocks"], "setup_s": setup_s,
        "h2d_probe_GBps": link,
    }
    if variants:
        var = {}
        var["reactive_on_demand"] = case(2, dims.k, True, h_all)
        var["sticky_per_layer_sets"] = case(dims.L, dims.k, False, h_all)
        # the same model on inputs shaped to the multi-stream routing statistics
        n_sh = warm + steps + 1
        tg = synth.route_targets(seed, dims, 1, n_sh)
        hs = torch.from_numpy(synth.shaped_hidden(seed, seed, dims, 1, tg).view(np.int16)).to(dev).view(torch.bfloat16)
        for name, pl, sl, rv in (("shaped_prefetch_shared_sets", 2, dims.k, False),
                                 ("shaped_sticky_per_layer_sets", dims.L, dims.k, False),
                                 ("shaped_reactive_on_demand", 2, dims.k, True)):
            r = case(pl, sl, rv, hs)
            r["routing"] = synth.routing_stats(tg[warm:warm + steps])
            var[name] = r
        # batch 8 with a least-recently-used cache of 32 experts per layer
        B = 8
        tg8 = synth.route_targets(seed, dims, B, n_sh)
        hs8 = torch.from_numpy(synth.shaped_hidden(seed, seed, dims, B, tg8).view(np.int16)).to(dev).view(torch.bfloat16)
        for name, pl, sl in (("shaped_b8_shared_sets", 2, 32), ("shaped_b8_lru_cache_32", dims.L, 32),
                             ("shaped_b8_lru_cache_64", dims.L, 64)):
            r = case(pl, sl, False, hs8, B=B)
            r["routing"] = synth.routing_stats(tg8[warm:warm + steps])
            var[name] = r
        out["variants"] = var
    return out, store


def run_multistream(args, dims, seed, ws, rank, local, batches=(8, 32, 64)):
    """Batched decode on inputs shaped to the pages' multi-stream routing statistics
    (next-token reuse ~0.44, Zipf popularity).  Algorithmic bytes come from the realised
    distinct experts of every layer and step."""
    import torch
    from synth.device import bf16_tensor
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    lys, hds = _load_model(dims, seed, dev)
    pk = peaks()
    res = {}
    warm, steps = 3, min(args.steps, 24)
    for B in batches:
        tg = synth.route_targets(seed, dims, B, warm + steps + 1)
        hs_np = synth.shaped_hidden(seed, seed, dims, B, tg)
        h_all = torch.from_numpy(hs_np.view(np.int16)).to(dev).view(torch.bfloat16)
        ctx = _context(dims, lys, hds, B)
        y = torch.empty((dims.L, B, dims.d), dtype=torch.bfloat16, device=dev)
        for t in range(warm):
            ctx.stack_decode(h_all[t], t, y_out=y)
        # per-step routing for the realised unique-expert bytes
        ctx.sync_status()
        idx_steps, exp_total = [], 0
        ms_sum = 0.0
        clocks = None
        launches = 0
        for t in range(warm, warm + steps):
            ms, clocks_t, l_t = _timed_steps(ctx, h_all, t, 1, y, ws, local)
            ms_sum += ms
            launches += l_t
            clocks = clocks_t if clocks is None else clocks
            idx, _ = ctx.get_routing(B)
            idx_steps.append(idx)
            exp_total += step_bytes(dims, idx, B)[0]
        # one uninterrupted timed region for the tokens/s figure
        ctx.close()
        ctx = _context(dims, lys, hds, B)
        for t in range(warm):
            ctx.stack_decode(h_all[t], t, y_out=y)
        ms_run, clk_run, l_run = _timed_steps(ctx, h_all, warm, steps, y, ws, local)
        ms_run = max_over_ranks(ms_run, ws)
        # end to end with host buffers
        h_host = h_all[warm:warm + steps].cpu().pin_memory()
        y_host = torch.empty((steps, dims.L, B, dims.d), dtype=torch.bfloat16, pin_memory=True)
        stream = torch.cuda.current_stream()
        ctx.stack_decode_host(h_host[0], warm + steps, y_host[0])   # untimed: allocates
        ctx.host_io_wait()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for t in range(steps):
            ctx.stack_decode_host(h_host[t], warm + steps + 1 + t, y_host[t])
        ctx.host_io_wait()
        b.record(stream)
        torch.cuda.synchronize()
        ms_e = max_over_ranks(a.elapsed_time(b), ws)
        ctx.close()
        tokens = sum_over_ranks(B * steps, ws)
        st = synth.routing_stats(np.stack(idx_steps))
        res[f"b{B}"] = {
            "value": tokens / (ms_run / 1e3), "unit": "tokens/s", "ms_per_step": ms_run / steps, "steps": steps,
            "batch": B, "path": ("phased kernels" if B <= 8 else
                                 f"phased kernels, {(B + 7) // 8} passes of up to 8 streams"),
            "gpu_launches": int(l_run), "clocks": clk_run,
            "routing": dict(st, matches_targets=bool(np.array_equal(np.sort(np.stack(idx_steps), -1),
                                                                    np.sort(tg[warm:warm + steps], -1)))),
            "roofline": _hbm_roofline(exp_total / steps, ms_run / steps, pk,
                                      "decode step (realised distinct experts of every layer + shared)"),
            "e2e": {"value": tokens / (ms_e / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h_host[0].numel() * 2),
                    "d2h_bytes_per_step": int(y_host[0].numel() * 2)},
        }
        del h_all
        _free_gpu()
    return res


def run_full_head_sweep(args, seed, ws, rank, local, ks=(2, 4, 8), H=256):
    """The prerouter head in its full form (fc1 -> erf-GELU -> fc2 plus the linear path, over
    u = [x; onehot(cur); onehot(prev)], width d + 2E) on the 40-layer model, at routing
    widths K = 2, 4, 8, one stream: tokens/s and HBM fraction on the expert bytes."""
    import torch
    import dataclasses
    dims0 = dataclasses.replace(synth.WORKLOADS["decode_b1_l40"]["dims"], head_hidden=H, head_onehot=1)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    lys, hds = _load_model(dims0, seed, dev)
    pk = peaks()
    out = {}
    steps, warm = min(args.steps, 32), 3
    for k in ks:
        dims = dataclasses.replace(dims0, k=k)
        ctx = _context(dims, lys, hds, 1)
        h_all = torch.stack([synth_hidden_tensor(seed, t, dims, 1, dev) for t in range(warm + steps)])
        y = torch.empty((dims.L, 1, dims.d), dtype=torch.bfloat16, device=dev)
        for t in range(warm):
            ctx.stack_decode(h_all[t], t, y_out=y)
        ms, clk, launches = _timed_steps(ctx, h_all, warm, steps, y, ws, local)
        ms = max_over_ranks(ms, ws)
        idx, _ = ctx.get_routing(1)
        exp_b = step_bytes(dims, idx, 1)[0]
        hb = 33 * (dims.E * dims.head_in + H * dims.head_in + dims.E * H) * 2
        out[f"k{k}"] = {"value": sum_over_ranks(steps, ws) / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms / steps,
                        "steps": steps, "top_k": k, "head_hidden": H, "head_input": dims.head_in,
                        "head_bytes_per_step": hb, "gpu_launches": int(launches), "clocks": clk,
                        "roofline": _hbm_roofline(exp_b, ms / steps, pk, "phased decode kernels (full heads)")}
        ctx.close()
        del h_all
    del lys, hds
    _free_gpu()
    return out


def synth_hidden_tensor(seed, t, dims, B, dev):
    from synth.device import bf16_tensor
    return bf16_tensor(synth.hidden(seed, t, dims.L, B, dims.d), dev)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--workload", default="decode_b1_l40")
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="only the named workload (default run adds the other workloads as sub-objects)")
    ap.add_argument("--decode-mode", type=int, default=0,
                    help="0 default, 1 one-launch, 2 graph, 3 eager per-layer, 4 phased")
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
    cpu = not args.no_cpu_baseline and rank == 0 and ws == 1
    if args.workload.startswith("stream"):
        out, _ = run_stream(args, dims, seed, ws, rank, local, variants=not args.no_extras)
        if rank == 0:
            print(json.dumps(out), flush=True)
        return
    if "tokens" in wl:
        out, ctx, _ = run_prefill(args, dims, seed, ws, rank, local)
        if cpu:
            import torch  # noqa: F401
            hs = synth.prefill_hidden(seed, 0, wl["tokens"], dims.d)[:256]
            out["cpu_baseline"] = cpu_baseline_tokens(dims, seed, hs, 0, dims.L, "256 of the chunk's 4096 tokens")
        if rank == 0:
            print(json.dumps(out), flush=True)
        ctx.close()
        return
    B = args.batch or (wl["batch"] if isinstance(wl.get("batch"), int) else 8)
    extras = not args.no_extras and ws == 1 and args.workload == "decode_b1_l40" and B == 1
    out, ctx = run_decode(args, dims, seed, B, ws, rank, local, extras)
    ctx.close()
    if cpu:
        out["cpu_baseline"] = cpu_baseline(dims, seed)
    if extras:
        # the other workloads of the same model family, each with its own timing, roofline,
        # clocks, end-to-end figure and CPU baseline
        _free_gpu()
        pargs = argparse.Namespace(**vars(args))
        pargs.steps, pargs.warmup = 3, 2
        pwl = synth.WORKLOADS["prefill_t4096_l40"]
        pre, pctx, _ = run_prefill(pargs, pwl["dims"], pwl["seed"], ws, rank, local)
        pctx.close()
        if cpu:
            hs = synth.prefill_hidden(pwl["seed"], 0, pwl["tokens"], dims.d)[:256]
            pre["cpu_baseline"] = cpu_baseline_tokens(pwl["dims"], pwl["seed"], hs, 0, dims.L,
                                                      "256 of the chunk's 4096 tokens")
        out["prefill_t4096_l40"] = pre
        _free_gpu()
        sargs = argparse.Namespace(**vars(args))
        sargs.steps, sargs.warmup = 16, 3
        swl = synth.WORKLOADS["stream_b1_l40"]
        st, store = run_stream(sargs, swl["dims"], swl["seed"], ws, rank, local, variants=True)
        del store
        if cpu:
            st["cpu_baseline"] = dict(out.get("cpu_baseline", {}), sample="the streaming tier computes exactly the "
                                      "resident decode step; its CPU baseline is the decode oracle's (this run)")
        out["stream_b1_l40"] = st
        _free_gpu()
        mwl = synth.WORKLOADS["decode_multistream_l40"]
        ms_res = run_multistream(args, mwl["dims"], mwl["seed"], ws, rank, local)
        if cpu:
            tg = synth.route_targets(mwl["seed"], mwl["dims"], 8, 1)
            hs8 = synth.shaped_hidden(mwl["seed"], mwl["seed"], mwl["dims"], 8, tg)
            ms_res["cpu_baseline"] = cpu_baseline_tokens(mwl["dims"], mwl["seed"], hs8[0, 0], 0, dims.L,
                                                         "one step of the batch-8 streams")
        out["decode_multistream_l40"] = ms_res
        _free_gpu()
        out["decode_b1_l40_full_head_k_sweep"] = run_full_head_sweep(args, seed, ws, rank, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
