"""Benchmark of the fused MoE layer (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode-fp8]
                    [--impl ours|reference] [--only-headline]

A step is one call of the whole layer (router, align, gather, w13 GEMM with
SiLU*up, [FP8 requantisation], w2 GEMM with router-weighted combine) on one
batch of synthetic tokens whose inputs already sit in HBM.  The headline
line times exactly K steps of the headline workload (default: decode-fp8,
the largest decode layer: T=64 H=7168 E=256 top_k=8 I=2048, E4M3 W8A8);
the key "workloads" carries the same fields for every one of the five layer
shapes (tiny, decode, decode-zipf, decode-fp8, prefill-zipf), each timed
over at least K steps and at least one second.  Each rank runs its own batch
(independent batches, weights replicated, no data-path collective): weak
scaling, value = all ranks' tokens / the slowest rank's device time.
Between timed steps L2 is flushed by writing a 256 MiB buffer; each step is
timed alone with CUDA events on the launch stream, and the flush is outside
the events.

Extra keys: us_per_layer, weight_bytes / weight_gbs (activated experts'
weight bytes counted once per step), stages_us (per-kernel-stage device time
from events the library records on the launch stream), roofline of the
dominant kernel (w13 grouped GEMM: weight bytes of the active experts / its
time vs the measured HBM peak at decode; 2 T k 2I H flops / its time vs the
measured bf16 peaks, burst and sustained, at prefill), e2e (same metric
through the host-buffer C-ABI call with the H2D/D2H copies in the timed
region), cpu_baseline (the fp64 oracle on a bounded token sample on the host
cores), gpu_launches and SM clocks sampled through NVML during each timed
region.

--impl reference times the fp64 CPU oracle (the only other implementation of
the layer; there is no installable reference package) on a bounded sample
per step, on rank 0 only.
"""
from __future__ import annotations

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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mixture_experts_layer_counts_b200.inputs import WORKLOADS, describe, make_inputs  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
HEADLINE = "decode-fp8"          # the largest decode layer
ORDER = ["decode-fp8", "tiny", "decode", "decode-zipf", "prefill-zipf"]
MIN_TIMED_S = 1.0                # each workload's timed region lasts at least this long
REF_SAMPLE_TOKENS = 1            # tokens per --impl reference step
CPU_BASELINE_TOKENS = 4          # tokens in the cpu_baseline sample
# Fallbacks when MEASURED_PEAKS.json is absent: an earlier measurement of this
# pool's B200s (HBM copy; cuBLAS bf16 GEMM burst and sustained under the power cap)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def peaks():
    """{hbm, bf16 burst, bf16 sustained, kind}: the measured figures of this
    pool's B200s when MEASURED_PEAKS.json is present, else the fallbacks."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        burst = float(d.get("bf16_tflops", d.get("bf16_tflops_sustained", FALLBACK_BF16_TFLOPS)))
        return dict(hbm=float(d["hbm_gbs"]), bf16=burst,
                    bf16_sustained=float(d.get("bf16_tflops_sustained", burst)), kind="measured")
    return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS, bf16_sustained=FALLBACK_BF16_TFLOPS_SUSTAINED,
                kind="fallback")


def kernel_traffic(workload):
    """ncu DRAM bytes per launch of the workload's roofline kernel, if captured
    for the current source of that kernel (the entry names its file)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(workload)
    if not d:
        return None
    src = os.path.join(ROOT, "mixture_experts_layer_counts_b200", "csrc", d.get("code_file", "gemm.cu"))
    if not os.path.exists(src) or code_sha(src) != d.get("code_sha"):
        return None
    return d.get("dram_bytes_per_launch")


def code_sha(path):
    """Hash of a C++ source without its // comments and blank lines (a
    comment edit leaves the captured counters valid; a code edit does not)."""
    lines = []
    for ln in open(path, encoding="utf-8"):
        code = ln.split("//", 1)[0].strip()
        if code:
            lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()[:16]


class ClockSampler:
    """SM clock and clock-event reasons of this rank's GPU, sampled through NVML
    every few milliseconds while the timed region runs (the GPU is found by
    its PCI bus id, so the NVML index need not match the CUDA index)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, dev, period_s=0.002):
        self.dev = dev
        self.period = period_s
        self.sm, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None

    def _handle(self):
        import pynvml

        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(self.dev)
        bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def _run(self, nv, h):
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        masks = [(n, getattr(nv, c, 0)) for n, c in self.REASONS]
        while not self._stop.is_set():
            try:
                self.sm.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                r = get_reasons(h)
                for n, m in masks:
                    if m and r & m:
                        self.reasons.add(n)
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        try:
            nv, h = self._handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self._thread = threading.Thread(target=self._run, args=(nv, h), daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=5)

    def summary(self):
        return {"sm_mhz": statistics.median(self.sm) if self.sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.sm)}


def dist_setup(n_gpus):
    """(rank, world, local rank) from the launcher's environment; one process
    per GPU over NCCL, or gloo on a host without GPUs (the CPU tests)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v, world):
    """Max of a per-rank float over all ranks (every rank gets it)."""
    if world == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_inputs(wl, dev, rank, world):
    """Each rank serves its own batch: rank-dependent hidden states, the same
    weights (same seed) on every rank."""
    inp = make_inputs(wl, dev, seed=wl["seed"])
    if world > 1:
        from mixture_experts_layer_counts_b200.inputs import make_hidden

        inp["hidden"] = make_hidden(wl, dev, seed=wl["seed"] + 1000 * rank)
    return inp


def whole_job_tokens_per_s(world, T, steps, max_total_ms):
    """Tokens all ranks processed / the slowest rank's device time."""
    return world * T * steps / (max_total_ms * 1e-3)


def oracle_sample_seconds(inp_host, wl, tokens):
    """Wall time of one oracle call on a bounded sample of the batch (inputs
    already on the host): the sampled tokens' rows form a layer call of their
    own (routing, per-tensor scales and every expert product of those tokens).
    The per-tensor FP8 scales then span the sample rather than the batch; the
    work per token is the same."""
    from oracle import moe_forward_ref

    hidden = inp_host["hidden"][list(tokens)]
    t0 = time.perf_counter()
    moe_forward_ref(hidden, inp_host["router_w"], inp_host["bias"], inp_host["w13"], inp_host["w2"],
                    wl["top_k"], wl["dtype"], inp_host["s13"], inp_host["s2"])
    return time.perf_counter() - t0


def host_copy(inp):
    from mixture_experts_layer_counts_b200.inputs import host_bits

    fp8 = inp["dtype"] == "fp8"
    return dict(hidden=host_bits(inp["hidden"]), router_w=host_bits(inp["router_w"]),
                bias=None if inp["router_bias"] is None else inp["router_bias"].float().cpu().numpy(),
                w13=host_bits(inp["w13"]), w2=host_bits(inp["w2"]),
                s13=inp["w13_scale"].cpu().numpy() if fp8 else None,
                s2=inp["w2_scale"].cpu().numpy() if fp8 else None)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [p.get("num_threads") for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_model():
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(wl, dev, seed=wl["seed"])
    host = host_copy(inp)
    del inp
    n_tok = min(REF_SAMPLE_TOKENS, wl["T"])
    samples = [[(i * n_tok + j) % wl["T"] for j in range(n_tok)] for i in range(args.warmup + args.steps)]
    for i in range(args.warmup):
        oracle_sample_seconds(host, wl, samples[i])
    times = [oracle_sample_seconds(host, wl, samples[args.warmup + i]) for i in range(args.steps)]
    total = sum(times)
    value = n_tok * args.steps / total
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": "MoE layer tokens/s", "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus if hasattr(args, "gpus") else 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload}: {describe(wl)}",
                   "sample": f"{n_tok} of {wl['T']} tokens per step"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "cpu": cpu_model(),
                         "kind": "oracle",
                         "sample": f"fp64 oracle; each step one token of the {args.workload} batch "
                                   f"(tokens 0, 1, 2, ... in turn) as a one-token layer call: its routing, "
                                   f"scales and its {wl['top_k']} experts' products"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


SWAP_MAX_TOKENS = 64   # the library's default swap-AB / normal threshold (tokens per expert)


def launches_per_step(wl, T):
    """Kernels one layer call launches: router (logits and top-k), the align
    (one grid, or two slice grids from T*k = 8192; with MOE_FUSE_ALIGN=1 the
    top-k's last CTA aligns decode-sized calls), gather, w13 and w2 GEMMs
    (one per orientation in use, or one fused launch for bf16 decode
    batches; the FP8 requantisation closes the last w13 launch), and the
    combine pass."""
    any_normal = T > SWAP_MAX_TOKENS and wl["H"] % 256 == 0
    A = T * wl["top_k"]
    fuse_align = os.environ.get("MOE_FUSE_ALIGN", "0") == "1" and A < 8192 and wl["E"] <= 256
    n_route = 2 + (0 if fuse_align else (2 if A >= 8192 else 1))
    # bf16 decode batches (T <= 32): both GEMMs in one launch; then the combine pass
    fused_ffn = wl["dtype"] == "bf16" and T <= 32 and os.environ.get("MOE_FUSED_FFN", "1") != "0"
    n_gemm = 1 if fused_ffn else 2 * (2 if any_normal else 1)
    return n_route + 1 + n_gemm + 1


def new_events(n, stream):
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for ev in evs:           # torch creates the CUDA event on first record
        ev.record(stream)
    return evs


def time_graph_steps(graph, flush, stream, steps, world, local):
    """Device time of `steps` replays of `graph`, each bracketed by events on
    `stream`, with an L2 flush before each (outside the events).  Returns
    (per-step ms list, max over ranks of the total ms, clock summary)."""
    tev = [new_events(2, stream) for _ in range(steps)]
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(steps):
            flush.zero_()
            tev[i][0].record(stream)
            graph.replay()
            tev[i][1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    step_ms = [a_.elapsed_time(b_) for a_, b_ in tev]
    return step_ms, max_over_ranks(sum(step_ms), world), clk.summary()


def measure_workload(name, wl, args, rank, world, local, steps_exact=None):
    """Every figure of one workload (see the module docstring).  steps_exact:
    time exactly that many steps; otherwise at least args.steps and at least
    MIN_TIMED_S of device time."""
    from mixture_experts_layer_counts_b200 import layer
    from mixture_experts_layer_counts_b200.layer import N_STAGE_EVENTS, STAGES

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    inp = rank_inputs(wl, dev, rank, world)
    T, H, E, I, k = inp["T"], inp["H"], inp["E"], inp["I"], inp["top_k"]
    dt = layer.dtype_code(inp["w13"])
    ws = layer.make_workspace(T, H, E, I, k, dt, dev)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    fwd = dict(w13_scale=inp["w13_scale"], w2_scale=inp["w2_scale"], out=out, workspace=ws)
    if args.batch_invariant:
        fwd["batch_invariant"] = True

    def call(**kw):
        layer.moe_forward(inp["hidden"], inp["router_w"], inp["router_bias"], inp["w13"], inp["w2"], k,
                          **fwd, **kw)

    # warm-up (the debug call also yields the routing this batch produces)
    dbg = {}
    call(debug=dbg)
    for _ in range(args.warmup):
        flush.zero_()
        call()
    torch.cuda.synchronize()
    code, info = layer.get_status(ws)
    if code != 0:
        raise RuntimeError(f"{name}: device status {code} info {info:#x} after warm-up")
    counts = dbg["counts"].cpu().numpy()
    e_act = int((counts > 0).sum())
    esize = 1 if dt == 1 else 2
    w13_bytes = e_act * 2 * I * H * esize
    w2_bytes = e_act * H * I * esize
    weight_bytes = w13_bytes + w2_bytes

    # The timed step is one replay of a CUDA graph holding one layer call, the
    # way an inference engine runs a layer (kernels chained by programmatic
    # dependent launch).
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for _ in range(3):
        flush.zero_()
        graph.replay()
    torch.cuda.synchronize()
    if steps_exact is not None:
        steps = steps_exact
    else:
        probe, _, _ = time_graph_steps(graph, flush, stream, 5, 1, local)
        per = max(statistics.median(probe), 1e-3) * 1e-3 + 40e-6     # + the flush
        steps = max(args.steps, int(math.ceil(MIN_TIMED_S / per)))
        steps = int(max_over_ranks(float(steps), world))
    step_ms, total_ms, clocks = time_graph_steps(graph, flush, stream, steps, world, local)
    code, info = layer.get_status(ws)
    if code != 0:
        raise RuntimeError(f"{name}: device status {code} info {info:#x} in the timed region")
    ms_per_step = total_ms / steps
    value = whole_job_tokens_per_s(world, T, steps, total_ms)
    del graph

    # Per-kernel breakdown: the same graph with the library's stage events
    # inside it (each event node costs ~2-3 us and breaks the programmatic
    # launch overlap, so these stage times are upper bounds).
    n_stage = min(steps, 300)
    gev = new_events(N_STAGE_EVENTS, stream)
    torch.cuda.synchronize()
    igraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(igraph):
        call(stage_events=gev)
    stage_sum = [0.0] * (N_STAGE_EVENTS - 1)
    for i in range(n_stage + 3):
        flush.zero_()
        igraph.replay()
        gev[-1].synchronize()
        if i >= 3:
            for st in range(1, N_STAGE_EVENTS):
                stage_sum[st - 1] += gev[st - 1].elapsed_time(gev[st])
    stage_ms = {STAGES[st]: stage_sum[st - 1] / n_stage for st in range(1, N_STAGE_EVENTS)}
    del igraph

    # The dominant kernel alone: a graph whose only stage events bracket the
    # w13 GEMM (entries 3 and 4).
    wev = new_events(2, stream)
    sel = [None] * N_STAGE_EVENTS
    sel[3], sel[4] = wev[0], wev[1]
    torch.cuda.synchronize()
    wgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(wgraph):
        call(stage_events=sel)
    w13_ms = []
    for i in range(n_stage + 3):
        flush.zero_()
        wgraph.replay()
        wev[1].synchronize()
        if i >= 3:
            w13_ms.append(wev[0].elapsed_time(wev[1]))
    del wgraph
    w13_kernel_ms = statistics.mean(w13_ms)

    # the same step launched directly (no graph): host launch gaps included
    n_direct = min(steps, 200)
    dev_ = [new_events(N_STAGE_EVENTS, stream) for _ in range(n_direct)]
    torch.cuda.synchronize()
    for i in range(n_direct):
        flush.zero_()
        call(stage_events=dev_[i])
    torch.cuda.synchronize()
    direct_ms = max_over_ranks(sum(e[0].elapsed_time(e[-1]) for e in dev_), world) / n_direct

    # end to end: pinned host hidden in, pinned host out, copies inside the timed region
    hin = inp["hidden"].cpu().pin_memory()
    hout = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(10, min(steps, 200))
    e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps)]
    barrier(world)
    torch.cuda.synchronize()
    dev_hidden = torch.empty_like(inp["hidden"])
    for i in range(e2e_steps):
        flush.zero_()
        e_ev[i][0].record(stream)
        if args.batch_invariant:   # no host-I/O entry point: the same copies around the call
            dev_hidden.copy_(hin, non_blocking=True)
            layer.moe_forward(dev_hidden, inp["router_w"], inp["router_bias"], inp["w13"], inp["w2"], k, **fwd)
            hout.copy_(out, non_blocking=True)
        else:
            layer.moe_forward_hostio(hin, inp["router_w"], inp["router_bias"], inp["w13"], inp["w2"], k,
                                     hout, ws, inp["w13_scale"], inp["w2_scale"])
        e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in e_ev), world)
    e2e_value = world * T * e2e_steps / (e2e_ms * 1e-3)

    # every algorithmic byte of the call: activated weights once, router
    # weights, hidden in, out, and the intermediates written and read once
    # (x in perm order, the intermediate h, the fp32 weighted slot rows)
    ab = esize
    all_bytes = (weight_bytes + E * H * 2 + T * H * 2 + T * H * 2 + 2 * T * k * H * ab +
                 2 * T * k * I * ab + 2 * T * k * H * 4)
    pk = peaks()
    w13_s = w13_kernel_ms * 1e-3
    flops = 2.0 * T * k * 3 * I * H
    # The w13 GEMM is the dominant kernel.  Decode batches (a few tokens per
    # expert, swap-AB tiles) are bound by streaming the activated experts'
    # weights: achieved = those bytes / time vs the measured HBM copy
    # bandwidth.  Prefill batches (normal-orientation tiles) are bound by the
    # tensor pipe: achieved = 2 T k 2I H / time vs the measured bf16 GEMM rate,
    # burst (the kernel timed on its own) and sustained (inside a long step).
    tensor_bound = T * k / max(e_act, 1) > SWAP_MAX_TOKENS
    w13_flops = 2.0 * T * k * 2 * I * H
    if tensor_bound:
        mult = 2.0 if dt == 1 else 1.0      # E4M3: the nominal fp8 / bf16 ratio
        ach = w13_flops / w13_s / 1e12
        pair = dt == 0 and I % 256 == 0 and os.environ.get("MOE_W13_2SM", "1") != "0"
        roof = {"kernel": "gemm_pair2sm_kernel<W13> (CTA pairs)" if pair else "grouped_gemm_kernel<normal, w13>",
                "bound": "tensor", "achieved": ach,
                "peak": mult * pk["bf16"], "unit": "TFLOP/s", "frac": ach / (mult * pk["bf16"]),
                "peak_kind": pk["kind"] + (" bf16 burst" if mult == 1 else " bf16 burst x 2 (fp8 nominal ratio)"),
                "peak_sustained": mult * pk["bf16_sustained"],
                "frac_of_sustained": ach / (mult * pk["bf16_sustained"]),
                "algorithmic_flops_per_launch": w13_flops}
        layer_frac = {"layer_tflops_frac_of_burst": flops / (ms_per_step * 1e-3) / 1e12 / (mult * pk["bf16"]),
                      "layer_tflops_frac_of_sustained":
                          flops / (ms_per_step * 1e-3) / 1e12 / (mult * pk["bf16_sustained"])}
    elif dt == 0 and T <= 32 and not args.batch_invariant and os.environ.get("MOE_FUSED_FFN", "1") != "0":
        # bf16 decode batches: gate/up and down GEMMs are one launch (ffn_swap_kernel);
        # the bracket covers it, its bytes are every activated weight byte
        achieved = weight_bytes / w13_s / 1e9
        roof = {"kernel": "ffn_swap_kernel (gate/up + down GEMMs, one launch)", "bound": "hbm",
                "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s", "frac": achieved / pk["hbm"],
                "peak_kind": pk["kind"], "algorithmic_bytes_per_launch": weight_bytes}
        layer_frac = {}
    else:
        achieved = w13_bytes / w13_s / 1e9
        roof = {"kernel": "grouped_gemm_kernel<swap-AB, w13>", "bound": "hbm", "achieved": achieved,
                "peak": pk["hbm"], "unit": "GB/s", "frac": achieved / pk["hbm"], "peak_kind": pk["kind"],
                "algorithmic_bytes_per_launch": w13_bytes}
        layer_frac = {}
    roof.update({"traffic": kernel_traffic(name), "kernel_us": 1e3 * w13_kernel_ms,
                 "timed_by": "CUDA events recorded on the launch stream right before and after the "
                             "w13 GEMM, inside a graph of the layer, L2 flushed per step"})
    res = {
        "workload": f"{name}: {describe(wl)}",
        "value": value, "unit": "tokens/s", "steps": steps, "ms_per_step": ms_per_step,
        "dtype": "fp8-e4m3" if dt == 1 else "bf16", "active_experts": e_act,
        "us_per_layer": 1e3 * ms_per_step,
        "us_per_layer_p50": 1e3 * statistics.median(step_ms),
        "us_per_layer_direct_launch": 1e3 * direct_ms,
        "weight_bytes": weight_bytes,
        "weight_gbs": weight_bytes / (ms_per_step * 1e-3) / 1e9,
        "weight_gbs_frac_of_hbm_peak": weight_bytes / (ms_per_step * 1e-3) / 1e9 / pk["hbm"],
        "weight_gbs_frac_of_8tbs": weight_bytes / (ms_per_step * 1e-3) / 8e12,
        "layer_tflops": flops / (ms_per_step * 1e-3) / 1e12, **layer_frac,
        "all_bytes": all_bytes, "all_gbs": all_bytes / (ms_per_step * 1e-3) / 1e9,
        "stages_us": {k_: 1e3 * v for k_, v in stage_ms.items()},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": T * H * 2,
                "d2h_bytes_per_step": T * H * 2, "steps": e2e_steps},
        "gpu_launches": launches_per_step(wl, T) * steps,
        "clocks": clocks,
    }
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and name == args.workload:
        host = host_copy(inp)
        toks = list(range(min(CPU_BASELINE_TOKENS, T)))
        secs = oracle_sample_seconds(host, wl, toks)
        cpu = {"value": len(toks) / secs, "unit": "tokens/s", "cores": blas_threads(), "cpu": cpu_model(),
               "kind": "oracle",
               "sample": f"fp64 oracle on tokens 0..{len(toks) - 1} of the batch as a layer call of their own "
                         f"(their routing, scales and expert products), {secs:.1f} s"}
    del inp, ws, out, flush
    torch.cuda.empty_cache()
    return res, cpu


ROPE_SHAPE = dict(T=16384, n_heads=32, head_dim=128, max_pos=8192)


def measure_inv_rope(local, steps=200):
    """Device time of the fused inverse-RoPE + per-head FP8 kernel on a
    prefill-sized call (inputs larger than L2, L2 flushed between steps).
    Algorithmic bytes: x read (2 B / element), codes written (1 B / element),
    one fp32 scale per head written, one table row pair read per token."""
    from mixture_experts_layer_counts_b200 import layer

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    T, nH, D, P = (ROPE_SHAPE[k] for k in ("T", "n_heads", "head_dim", "max_pos"))
    g = torch.Generator(device=dev).manual_seed(11)
    x = torch.randn(T, nH, D, generator=g, device=dev).to(torch.bfloat16)
    pos = torch.randint(0, P, (T,), generator=g, device=dev, dtype=torch.int32)
    ang = torch.arange(P, device=dev, dtype=torch.float64)[:, None] * \
        (10000.0 ** (-torch.arange(D // 2, device=dev, dtype=torch.float64) * 2.0 / D))[None, :]
    ct, st = torch.cos(ang).float().contiguous(), torch.sin(ang).float().contiguous()
    codes = torch.empty(T, nH, D, dtype=torch.uint8, device=dev)
    scales = torch.empty(T, nH, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for _ in range(5):
        layer.inv_rope_fp8_quant(x, pos, ct, st, codes, scales)
    ev = [new_events(2, stream) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        layer.inv_rope_fp8_quant(x, pos, ct, st, codes, scales)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    nbytes = T * nH * D * 3 + T * nH * 4 + T * D * 4 + T * 4
    pk = peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"shape": dict(ROPE_SHAPE), "us": 1e3 * ms, "algorithmic_bytes": nbytes,
            "roofline": {"kernel": "inv_rope_fp8_kernel", "bound": "hbm", "achieved": gbs, "peak": pk["hbm"],
                         "unit": "GB/s", "frac": gbs / pk["hbm"], "peak_kind": pk["kind"]},
            "tokens_per_s": T / (ms * 1e-3), "steps": steps}


def sweep_orientation(local, counts=(8, 16, 24, 32, 48, 64, 80, 96, 128, 160, 192, 256), reps=20):
    """Gate/up and down GEMM time under forced swap-AB and forced normal
    orientation, for E = 16 experts holding exactly c tokens each (a one-hot
    router sends token t to expert t mod 16, top_k = 1), H = 4096, I = 1536,
    bf16.  Each GEMM timed by the library's stage events, L2 flushed before
    every call; median of `reps` calls.  One JSON line per c."""
    from mixture_experts_layer_counts_b200 import layer

    H, I, E, k = 4096, 1536, 16, 1
    dev = torch.device("cuda", local)
    g = torch.Generator(device=dev).manual_seed(0)
    w13 = (torch.randn(E, 2 * I, H, generator=g, device=dev) * 0.02).to(torch.bfloat16)
    w2 = (torch.randn(E, H, I, generator=g, device=dev) * 0.02).to(torch.bfloat16)
    router_w = torch.zeros(E, H, device=dev)
    router_w[torch.arange(E), torch.arange(E)] = 1.0
    router_w = router_w.to(torch.bfloat16)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for c in counts:
        T = E * c
        hidden = torch.randn(T, H, generator=g, device=dev) * 0.1
        hidden[:, :E] = 0.0
        idx = torch.arange(T, device=dev)
        hidden[idx, idx % E] = 8.0
        hidden = hidden.to(torch.bfloat16)
        ws = layer.make_workspace(T, H, E, I, k, 0, dev)
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        row = {"tokens_per_expert": c}
        for force, name in ((1, "swap"), (2, "normal")):
            evs = new_events(8, torch.cuda.current_stream(dev))
            t13, t2 = [], []
            for it in range(reps + 3):
                flush.zero_()
                layer.moe_forward(hidden, router_w, None, w13, w2, k, out=out, workspace=ws, force_orient=force,
                                  stage_events=evs)
                torch.cuda.synchronize()
                if it >= 3:
                    t13.append(evs[3].elapsed_time(evs[4]) * 1e3)
                    t2.append(evs[5].elapsed_time(evs[6]) * 1e3)
            dbg = {}
            layer.moe_forward(hidden, router_w, None, w13, w2, k, debug=dbg)
            cnt = dbg["counts"].cpu()
            assert int(cnt.min()) == c and int(cnt.max()) == c, "routing did not give c tokens per expert"
            row[name + "_w13_us"] = statistics.median(t13)
            row[name + "_w2_us"] = statistics.median(t2)
        print(json.dumps(row), flush=True)


def route_only(wl, local, steps=200):
    """Device time of the router alone (moe_route: logits and top-k) on the
    workload's hidden states and router weights; no expert weights are
    allocated (small enough for full-set profiler captures).  One JSON line."""
    from mixture_experts_layer_counts_b200 import layer
    from mixture_experts_layer_counts_b200.inputs import make_hidden, make_router, zipf_bias

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    hidden, router_w = make_hidden(wl, dev), make_router(wl, dev)
    bias = zipf_bias(wl["E"]).to(dev) if wl["zipf"] else None
    ws = layer.make_workspace(wl["T"], wl["H"], wl["E"], 128, wl["top_k"], 0, dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for _ in range(5):
        layer.moe_route(hidden, router_w, bias, wl["top_k"], workspace=ws)
    ev = [new_events(2, stream) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        layer.moe_route(hidden, router_w, bias, wl["top_k"], workspace=ws)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    us = 1e3 * statistics.median(a.elapsed_time(b) for a, b in ev)
    print(json.dumps({"route_only": describe(wl), "us": us, "steps": steps}), flush=True)


def run_ours(args, wl, rank, world, local):
    pk = peaks()
    head, cpu = measure_workload(args.workload, wl, args, rank, world, local, steps_exact=args.steps)
    nested = {}
    if world == 1 and not args.only_headline:
        for name in ORDER:
            if name == args.workload:
                nested[name] = head
                continue
            w = dict(WORKLOADS[name])
            nested[name] = measure_workload(name, w, args, rank, world, local)[0]
    line = {
        "metric": "MoE layer tokens/s", "value": head["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": head["dtype"], "data": "synthetic",
        "config": {"workload": head["workload"], "global_batch": world * wl["T"],
                   "active_experts": head["active_experts"],
                   "l2": "flushed (256 MiB write) between timed steps",
                   "parallelism": f"dp{world} (independent batches)",
                   "mode": "batch_invariant" if args.batch_invariant else "default"},
        "timing": "per step: device time of one CUDA-graph replay of moe_forward (events on the "
                  "stream around the replay); stages_us from a separate instrumented graph",
        "peaks": pk,
    }
    for key in ("us_per_layer", "us_per_layer_p50", "us_per_layer_direct_launch", "weight_bytes", "weight_gbs",
                "weight_gbs_frac_of_hbm_peak", "weight_gbs_frac_of_8tbs", "layer_tflops", "all_bytes",
                "all_gbs", "stages_us", "roofline", "e2e", "gpu_launches", "clocks"):
        line[key] = head[key]
    if nested:
        line["workloads"] = nested
        line["inv_rope_fp8"] = measure_inv_rope(local)
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps of the headline (default 200; "
                                                             "reference: 5)")
    ap.add_argument("--warmup", type=int, default=None, help="warm-up steps (default 10; reference: 1)")
    ap.add_argument("--workload", default=HEADLINE, choices=list(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--only-headline", action="store_true", help="skip the other workloads")
    ap.add_argument("--rope-only", action="store_true",
                    help="time the fused inverse-RoPE + FP8 kernel alone (one JSON line)")
    ap.add_argument("--route-only", action="store_true",
                    help="time the router alone on the workload's hidden states (no expert weights)")
    ap.add_argument("--sweep-orientation", action="store_true",
                    help="time both GEMMs under forced swap-AB / normal orientation over tokens per expert")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch-invariant", action="store_true",
                    help="time moe_forward_batch_invariant (bf16 workloads)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T of the workload (smaller cases for profiler captures)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E of the workload (smaller cases for profiler captures)")
    args = ap.parse_args()
    wl = dict(WORKLOADS[args.workload])
    if args.tokens:
        wl["T"] = args.tokens
    if args.experts:
        wl["E"] = args.experts
    if args.tokens or args.experts or args.batch_invariant:
        args.only_headline = True
    if args.impl == "reference":
        # the fp64 oracle takes seconds per token: small defaults, one-token samples
        args.steps = 5 if args.steps is None else args.steps
        args.warmup = 1 if args.warmup is None else args.warmup
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        run_reference(args, wl, rank, world)
        return
    args.steps = 200 if args.steps is None else args.steps
    args.warmup = 10 if args.warmup is None else args.warmup
    rank, world, local = dist_setup(args.gpus)
    if args.sweep_orientation:
        sweep_orientation(local)
        return
    if args.route_only:
        route_only(wl, local, args.steps)
        return
    if args.rope_only:
        print(json.dumps({"inv_rope_fp8": measure_inv_rope(local, args.steps)}), flush=True)
        return
    try:
        run_ours(args, wl, rank, world, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
