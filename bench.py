"""Benchmark of the fused MoE layer (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode] [--impl ours|reference]

A step is one call of the whole layer (router, align, gather, w13 GEMM with
SiLU*up, [FP8 requant], w2 GEMM with router-weighted slot scatter, combine)
on one batch of synthetic decode tokens whose inputs already sit in HBM.
Each rank runs its own batch (independent decode batches, weights replicated,
no data-path collective): weak scaling, value = all ranks' tokens / the
slowest rank's device time.  Between timed steps L2 is flushed by writing a
256 MiB buffer; each step is timed alone with CUDA events on the launch
stream, and the flush is outside the events.

Extra keys: us_per_layer, weight_bytes / weight_gbs (activated experts'
weight bytes counted once per step), stages_us (per-kernel-stage device time
from events the library records on the launch stream), roofline of the
dominant kernel (w13 grouped GEMM, weight bytes of active experts / its
measured time vs the measured HBM peak), e2e (same metric through the
host-buffer C-ABI call with the H2D/D2H copies in the timed region),
cpu_baseline (the fp64 oracle on a bounded token sample on the host cores),
gpu_launches and clocks sampled with nvidia-smi during the timed region.

--impl reference times the fp64 CPU oracle (the only other implementation of
the layer; there is no installable reference package) on a bounded token
sample per step, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mixture_experts_layer_counts_b200.inputs import WORKLOADS, describe, make_inputs  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
REF_SAMPLE_TOKENS = 1          # tokens per --impl reference step
CPU_BASELINE_TOKENS = 4        # tokens in the cpu_baseline sample
FALLBACK_HBM_GBS = 6650.0


FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def peaks():
    """(HBM GB/s, dense bf16 TFLOP/s sustained, kind): the driver's measured figures."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops_sustained", d.get("bf16_tflops"))), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


def kernel_traffic(workload):
    """ncu DRAM bytes per launch of the w13 kernel, if captured for this source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(workload)
    if not d:
        return None
    if code_sha(os.path.join(ROOT, "mixture_experts_layer_counts_b200", "csrc", "gemm.cu")) != d.get("gemm_cu_sha"):
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
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, dev):
        self.dev = dev
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


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
    """Wall time of one oracle call on a token sample (inputs already on host)."""
    from oracle import moe_forward_ref

    t0 = time.perf_counter()
    moe_forward_ref(inp_host["hidden"], inp_host["router_w"], inp_host["bias"], inp_host["w13"],
                    inp_host["w2"], wl["top_k"], wl["dtype"], inp_host["s13"], inp_host["s2"],
                    tokens=tokens)
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
    toks = list(range(REF_SAMPLE_TOKENS))
    for _ in range(args.warmup):
        oracle_sample_seconds(host, wl, toks)
    times = [oracle_sample_seconds(host, wl, toks) for _ in range(args.steps)]
    total = sum(times)
    value = len(toks) * args.steps / total
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": "MoE layer tokens/s", "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload}: {describe(wl)}", "sample": f"{len(toks)} of {wl['T']} tokens"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "cpu": cpu_model(),
                         "kind": "oracle",
                         "sample": f"fp64 oracle, tokens 0..{len(toks) - 1} of the {args.workload} batch "
                                   f"(full routing of all {wl['T']} tokens) per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


SWAP_MAX_TOKENS = 64   # the library's default swap-AB / normal threshold (tokens per expert)


def launches_per_step(wl, T):
    """Kernels one layer call launches: router (logits, top-k), align (two
    slice grids from T*k = 8192 on), gather, w13 and w2 GEMMs (one per
    orientation in use), FP8 requant, combine."""
    any_normal = T > SWAP_MAX_TOKENS and wl["H"] % 256 == 0
    n_align = 2 if T * wl["top_k"] >= 8192 else 1
    n = 2 + n_align + 1 + 2 * (2 if any_normal else 1) + 1
    return n + (1 if wl["dtype"] == "fp8" else 0)


def run_ours(args, wl, rank, world, local):
    from mixture_experts_layer_counts_b200 import layer

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

    def step(events=None):
        layer.moe_forward(inp["hidden"], inp["router_w"], inp["router_bias"], inp["w13"], inp["w2"], k,
                          stage_events=events, **fwd)

    # warm-up (also yields the routing this batch produces)
    dbg = {}
    layer.moe_forward(inp["hidden"], inp["router_w"], inp["router_bias"], inp["w13"], inp["w2"], k,
                      debug=dbg, **fwd)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    code, info = layer.get_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} info {info:#x} after warm-up")
    counts = dbg["counts"].cpu().numpy()
    e_act = int((counts > 0).sum())
    esize = 1 if dt == 1 else 2
    w13_bytes = e_act * 2 * I * H * esize
    w2_bytes = e_act * H * I * esize
    weight_bytes = w13_bytes + w2_bytes

    from mixture_experts_layer_counts_b200.layer import N_STAGE_EVENTS, STAGES

    def new_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for ev in evs:           # torch creates the CUDA event on first record
            ev.record(stream)
        return evs

    # The timed step is one replay of a CUDA graph holding one layer call, the
    # way a decode engine runs it (kernels chained by programmatic dependent
    # launch).  Start/end events are recorded on the stream around each
    # replay; the L2 flush sits between steps, outside the events.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(3):
        flush.zero_()
        graph.replay()
    tev = [new_events(2) for _ in range(args.steps)]
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            tev[i][0].record(stream)
            graph.replay()
            tev[i][1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    code, info = layer.get_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} info {info:#x} in the timed region")
    step_ms = [a_.elapsed_time(b_) for a_, b_ in tev]
    total_ms = max_over_ranks(sum(step_ms), world)
    ms_per_step = total_ms / args.steps
    value = whole_job_tokens_per_s(world, T, args.steps, total_ms)
    del graph

    # Per-kernel breakdown: the same graph with the library's 8 stage events
    # recorded inside it (each event node costs ~2-3 us, so these stage times
    # are upper bounds and their sum exceeds the step time above).
    gev = new_events(N_STAGE_EVENTS)
    torch.cuda.synchronize()
    igraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(igraph):
        step(gev)
    n_stage = min(args.steps, 1000)
    stage_sum = [0.0] * (N_STAGE_EVENTS - 1)
    for i in range(n_stage + 3):
        flush.zero_()
        igraph.replay()
        gev[-1].synchronize()
        if i >= 3:
            for s in range(1, N_STAGE_EVENTS):
                stage_sum[s - 1] += gev[s - 1].elapsed_time(gev[s])
    stage_ms = {STAGES[s]: stage_sum[s - 1] / n_stage for s in range(1, N_STAGE_EVENTS)}
    del igraph

    # The dominant kernel alone: a graph whose only stage events bracket the
    # w13 GEMM (entries 3 and 4), so the kernel is timed with one event node
    # on each side instead of eight.
    wev = new_events(2)
    sel = [None] * N_STAGE_EVENTS
    sel[3], sel[4] = wev[0], wev[1]
    torch.cuda.synchronize()
    wgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(wgraph):
        layer.moe_forward(inp["hidden"], inp["router_w"], inp["router_bias"], inp["w13"], inp["w2"], k,
                          stage_events=sel, **fwd)
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
    n_direct = min(args.steps, 500)
    dev_ = [new_events(N_STAGE_EVENTS) for _ in range(n_direct)]
    torch.cuda.synchronize()
    for i in range(n_direct):
        flush.zero_()
        step(dev_[i])
    torch.cuda.synchronize()
    direct_ms = max_over_ranks(sum(e[0].elapsed_time(e[-1]) for e in dev_), world) / n_direct

    # end to end: pinned host hidden in, pinned host out, copies inside the timed region
    hin = inp["hidden"].cpu().pin_memory()
    hout = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(10, min(args.steps, 200))
    e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps)]
    barrier(world)
    torch.cuda.synchronize()
    dev_hidden = torch.empty_like(inp["hidden"])
    for i in range(e2e_steps):
        flush.zero_()
        e_ev[i][0].record(stream)
        if args.batch_invariant:   # no host-I/O entry point: the same copies around the call
            dev_hidden.copy_(hin, non_blocking=True)
            layer.moe_forward(dev_hidden, inp["router_w"], inp["router_bias"], inp["w13"], inp["w2"], k,
                              **fwd)
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
    peak, peak_tf, peak_kind = peaks()
    w13_s = w13_kernel_ms * 1e-3
    # The w13 GEMM bracket is the dominant kernel.  Decode batches (a few
    # tokens per expert, swap-AB tiles) are bound by streaming the activated
    # experts' weights: achieved = those bytes / time vs the measured HBM
    # copy bandwidth.  Prefill batches (normal-orientation tiles) are bound by
    # the tensor pipe: achieved = 2 * T*k * 2I * H / time vs the measured
    # sustained bf16 GEMM rate (the kernel runs inside a long step).
    tensor_bound = T * k / max(e_act, 1) > 64
    w13_flops = 2.0 * T * k * 2 * I * H
    if tensor_bound:
        roof = {"kernel": "grouped_gemm_kernel<normal, w13>", "bound": "tensor",
                "achieved": w13_flops / w13_s / 1e12, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": w13_flops / w13_s / 1e12 / peak_tf, "peak_kind": peak_kind + " (bf16, sustained)",
                "algorithmic_flops_per_launch": w13_flops}
        if dt == 1:
            roof["peak"] = 2 * peak_tf
            roof["frac"] = roof["achieved"] / roof["peak"]
            roof["peak_kind"] = peak_kind + " (bf16 sustained x 2, the nominal fp8/bf16 ratio)"
    else:
        achieved = w13_bytes / w13_s / 1e9
        roof = {"kernel": "grouped_gemm_kernel<swap-AB, w13>", "bound": "hbm", "achieved": achieved,
                "peak": peak, "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind,
                "algorithmic_bytes_per_launch": w13_bytes}
    roof.update({"traffic": kernel_traffic(args.workload), "kernel_us": 1e3 * w13_kernel_ms,
                 "timed_by": "CUDA events recorded on the launch stream right before and after the "
                             "w13 GEMM, inside a graph of the layer, L2 flushed per step"})
    line = {
        "metric": "MoE layer tokens/s", "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8-e4m3" if dt == 1 else "bf16", "data": "synthetic",
        "config": {"workload": f"{args.workload}: {describe(wl)}", "global_batch": world * T,
                   "active_experts": e_act, "l2": "flushed (256 MiB write) between timed steps",
                   "parallelism": f"dp{world} (independent decode batches)",
                   "mode": "batch_invariant" if args.batch_invariant else "default"},
        "us_per_layer": 1e3 * ms_per_step,
        "us_per_layer_p50": 1e3 * statistics.median(step_ms),
        "us_per_layer_direct_launch": 1e3 * direct_ms,
        "timing": "per step: device time of one CUDA-graph replay of moe_forward (events on the "
                  "stream around the replay); stages_us from a separate instrumented graph",
        "weight_bytes": weight_bytes,
        "weight_gbs": weight_bytes / (ms_per_step * 1e-3) / 1e9,
        "weight_gbs_frac_of_measured_hbm": weight_bytes / (ms_per_step * 1e-3) / 1e9 / peak,
        "weight_gbs_frac_of_8tbs": weight_bytes / (ms_per_step * 1e-3) / 8e12,
        "layer_tflops": 2.0 * T * k * 3 * I * H / (ms_per_step * 1e-3) / 1e12,
        "all_bytes": all_bytes,
        "all_gbs": all_bytes / (ms_per_step * 1e-3) / 1e9,
        "stages_us": {k_: 1e3 * v for k_, v in stage_ms.items()},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": T * H * 2,
                "d2h_bytes_per_step": T * H * 2, "steps": e2e_steps},
        "gpu_launches": launches_per_step(wl, T) * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = host_copy(inp)
        toks = list(range(min(CPU_BASELINE_TOKENS, T)))
        secs = oracle_sample_seconds(host, wl, toks)
        line["cpu_baseline"] = {"value": len(toks) / secs, "unit": "tokens/s", "cores": blas_threads(),
                                "cpu": cpu_model(),
                                "kind": "oracle",
                                "sample": f"fp64 oracle on tokens 0..{len(toks) - 1} of the batch "
                                          f"(routing of all {T} tokens), {secs:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default 5000; reference: 5)")
    ap.add_argument("--warmup", type=int, default=None, help="warm-up steps (default 20; reference: 1)")
    ap.add_argument("--workload", default="decode", choices=list(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
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
    if args.impl == "reference":
        # the fp64 oracle takes seconds per token: small defaults, one-token samples
        args.steps = 5 if args.steps is None else args.steps
        args.warmup = 1 if args.warmup is None else args.warmup
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        run_reference(args, wl, rank, world)
        return
    args.steps = 5000 if args.steps is None else args.steps
    args.warmup = 20 if args.warmup is None else args.warmup
    rank, world, local = dist_setup(args.gpus)
    try:
        run_ours(args, wl, rank, world, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
