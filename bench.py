"""Benchmark of the pre-gated mixture-of-LoRA hot path (one JSON line on rank 0).

A step is one pass of the whole path over one batch of synthetic tokens:
router + top-k + gates (once), segments (once), then the SGMM shrink/expand
fused into the base-output add for every (layer, shared-input group) of the
workload.  The headline workload is ``prefill`` (Llama-2-7B layer set, 8192
tokens, 16 rank-16 adapters with Zipf(1.1) popularity, top-2); the other
full-size workloads (decode, multitenant, merge) are timed in the same run and
reported under ``workloads``, and so is ``prefill_fused``: the prefill layers
with their base projections, each call the base GEMM and the adapters in one
contraction (apr_linear_lora), beside the unfused pipeline it replaces (a
library GEMM, then the SGMM add), and ``merge_crossover``: for 1-8 tokens that
share one routing, the steps after which an in-place merge (with its exact
unmerge) beats adding the adapters unmerged.  Each step is captured once in a CUDA graph
and replayed; ``e2e`` times the eager C-ABI calls with the step's activations
copied in from and out to pinned host memory.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--also decode,multitenant,merge,prefill_fused,merge_crossover|none]
                    [--impl reference]

With N > 1 (torchrun, one process per GPU) every rank runs its own batch
(weak scaling: tokens are independent and the path has no exchange step);
timing is the max over ranks of the CUDA-event time.
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

METRIC = "mixture-of-LoRA SGMM tokens/s at 1 B200; % of HBM / tensor-core roofline"
W_CONFIG_LAYERS = {"tiny": 4, "decode": 32, "prefill": 32, "multitenant": 32, "merge": 32}
DESCR = {
    "decode": "decode: Llama-2-7B layer set (32 layers; q,k,v,o 4096->4096; gate,up 4096->11008; "
              "down 11008->4096), 8 adapters rank 16, top-2 pre-gate, 32 tokens/step, uniform, bf16",
    "prefill": "prefill: same layers, 16 adapters rank 16, top-2, 8192 tokens, Zipf(1.1) popularity, bf16",
    "multitenant": "multi-tenant: 32 layers q,v 4096->4096, 256 adapters ranks {8,16,32,64}, top-1, "
                   "4096 tokens uniform, bf16",
    "merge": "batch-1 merge: 224 decode-shaped weights, top-2 merged W' = W + sum g B A in one launch, "
             "then one GEMV per weight, bf16",
    "tiny": "tiny: 4 layers x 256->256, 8 adapters rank 8, top-2, 64 tokens, fp32",
    "prefill_fused": "prefill with the base projections: every layer call is y = x W^T + sum g B A x in one "
                     "contraction (apr_linear_lora), same layers, adapters and routing as prefill, bf16",
}
# workloads that are another workload's configuration run in another mode
BASE_MODE = {"prefill_fused": ("prefill", "fused")}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _code_tokens(text):
    """C/CUDA source without comments and with whitespace runs collapsed: edits to comments or
    layout leave it unchanged, any change to the code does not."""
    import re
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"':                                   # string literal (inline PTX), kept verbatim
            j = i + 1
            while j < n and text[j] != '"':
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
            out.append(c)
            i += 1
    return re.sub(r"\s+", " ", "".join(out)).strip()


def kernel_source_hash():
    """SHA-1 prefix over the kernel sources' code (comments and layout ignored), matched against
    the one a DRAM capture was taken on."""
    import glob
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "adapter_pregate_router_b200", "csrc")
    for f in sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))):
        h.update(os.path.basename(f).encode())
        with open(f, encoding="utf-8") as fh:
            h.update(_code_tokens(fh.read()).encode())
    return h.hexdigest()[:16]


TRAFFIC_FILE = os.path.join("profiles", "dram_traffic.json")


def measured_traffic(workload):
    """DRAM bytes per SGMM call from the committed ncu capture, or None when the kernels changed
    since (the capture records the kernel-source hash it was taken on)."""
    path = os.path.join(ROOT, TRAFFIC_FILE)
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    ent = d.get("workloads", {}).get(workload)
    if not ent or ent.get("kernel_source_hash") != kernel_source_hash():
        return None
    return float(ent["bytes_per_call"])


def ingest_traffic(csv_path, workload, calls, command, kernels=None, last=0):
    """Record an ncu launch capture (``--metrics dram__bytes_read.sum,dram__bytes_write.sum``,
    ``--csv``) as the DRAM bytes per SGMM call of ``workload``: the sum over the captured launches
    (those whose kernel name matches the regex ``kernels``, the last ``last`` of them when given)
    divided by ``calls``, keyed to the current kernel-source hash."""
    import csv
    import re
    with open(csv_path) as f:
        rows = [r for r in csv.reader(l for l in f if l.startswith('"'))]
    head = rows[0]
    im, iv, iu = head.index("Metric Name"), head.index("Metric Value"), head.index("Metric Unit")
    ik, iid = head.index("Kernel Name"), head.index("ID")
    scale = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    per_launch = {}
    for r in rows[1:]:
        if kernels and not re.search(kernels, r[ik]):
            continue
        if r[im] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            per_launch[int(r[iid])] = per_launch.get(int(r[iid]), 0.0) + float(r[iv].replace(",", "")) * scale.get(r[iu], 1.0)
    ids = sorted(per_launch)
    if last:
        ids = ids[-last:]
    tot = sum(per_launch[i] for i in ids)
    path = os.path.join(ROOT, TRAFFIC_FILE)
    d = {"note": "DRAM bytes per SGMM call from ncu launch captures (dram__bytes_read.sum + "
                 "dram__bytes_write.sum over the captured launches / calls); written by bench.py --ingest-traffic",
         "workloads": {}}
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
    d["workloads"][workload] = {"bytes_per_call": tot / calls, "calls": calls, "kernel_source_hash": kernel_source_hash(),
                                "command": command}
    with open(path, "w") as f:
        json.dump(d, f, indent=1, sort_keys=True)
        f.write("\n")
    return tot / calls


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        if not self.lines:
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value, world, device=None):
    """Largest value over all ranks (the job's wall time is its slowest rank's)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    if device is None:
        device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank, ms_local, world, device=None):
    """Whole-job throughput: units processed by all ranks / the slowest rank's time."""
    ms = max_over_ranks(ms_local, world, device)
    return units_per_rank * world / (ms / 1e3), ms


# ---------------------------------------------------------------- CPU oracle leg


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OracleSample:
    """The fp64 oracle on a bounded sample of one step of ``cfg``.

    Inputs of the first ``n_layers`` layers are prepared once, outside the
    clock; one pass times the route + segments over all tokens and those
    layers (every projection, every token), and the step time is scaled to
    all layers.  BLAS may use ``threads`` threads (the oracle's per-token loop
    itself is plain Python on one core).
    """

    def __init__(self, cfg, layer_budget_s):
        from adapter_pregate_router_b200 import workloads as W
        from oracle import apr_oracle as O
        self.cfg, self.W, self.O = cfg, W, O
        self.ranks = W.ranks(cfg)
        self.h, self.Wr, _ = W.router_inputs(cfg)
        idx, gate, _ = O.pregate_route(self.h, self.Wr, cfg.k)
        self.sel = set(idx.reshape(-1).tolist())
        self.layers = [self._prepare(0)]
        t = self._time_layer(self.layers[0], idx, gate)
        n = int(max(1, min(cfg.layers, layer_budget_s / max(t, 1e-6))))
        for l in range(1, n):
            self.layers.append(self._prepare(l))

    def _prepare(self, l):
        cfg, W = self.cfg, self.W
        items = []
        for g in cfg.groups:
            if cfg.merge:
                for p, d_out in zip(g.proj_names, g.d_outs):
                    Wt = W.host_tensor(cfg, W.w_key(l, g.name, p), (d_out, g.d_in))
                    A = [W.host_tensor(cfg, W.a_key(l, g.name, p, e), (int(self.ranks[e]), g.d_in))
                         if e in self.sel else None for e in range(cfg.E)]
                    B = [W.host_tensor(cfg, W.b_key(l, g.name, p, e), (d_out, int(self.ranks[e])))
                         if e in self.sel else None for e in range(cfg.E)]
                    items.append(("merge", Wt, A, B, W.host_tensor(cfg, W.xm_key(l, g.name, p), (g.d_in,))))
                continue
            x = W.host_tensor(cfg, W.x_key(l, g.name), (cfg.T, g.d_in))
            for p, d_out in zip(g.proj_names, g.d_outs):
                A = [W.host_tensor(cfg, W.a_key(l, g.name, p, e), (int(self.ranks[e]), g.d_in))
                     if e in self.sel else None for e in range(cfg.E)]
                B = [W.host_tensor(cfg, W.b_key(l, g.name, p, e), (d_out, int(self.ranks[e])))
                     if e in self.sel else None for e in range(cfg.E)]
                yb = W.host_tensor(cfg, W.ybase_key(l, g.name, p), (cfg.T, d_out))
                items.append(("sgmm", x, A, B, yb))
        return items

    def _time_layer(self, items, idx, gate):
        O = self.O
        t0 = time.perf_counter()
        for it in items:
            if it[0] == "merge":
                _, Wt, A, B, xv = it
                O.gemv(O.merge_adapters(Wt, A, B, idx[0], gate[0]), xv)
            else:
                _, x, A, B, yb = it
                O.sgmm_shrink_expand(x, A, B, idx, gate, yb)
        return time.perf_counter() - t0

    def step_seconds(self, threads=1):
        from threadpoolctl import threadpool_limits
        O, cfg = self.O, self.cfg
        with threadpool_limits(limits=threads):
            t0 = time.perf_counter()
            idx, gate, _ = O.pregate_route(self.h, self.Wr, cfg.k)
            O.segment_tokens(idx, cfg.E)
            t_route = time.perf_counter() - t0
            t_layers = sum(self._time_layer(items, idx, gate) for items in self.layers)
        return t_route + t_layers * cfg.layers / len(self.layers)

    def describe(self, threads):
        c = self.cfg
        return (f"route+segments over all {c.T} tokens plus {len(self.layers)} of {c.layers} layers "
                f"(every projection and token) timed, scaled to {c.layers} layers; fp64 numpy oracle, "
                f"BLAS on {threads} thread(s), the per-token loop in one Python thread")


def cpu_baseline(cfg, budget_s):
    """Oracle passes for about ``budget_s`` seconds of CPU work, with BLAS on all host cores and,
    beside it, on one thread."""
    smp = OracleSample(cfg, layer_budget_s=budget_s / 6)
    cores = host_cores()
    out = {}
    for threads in (cores, 1):
        times, spent = [], 0.0
        while spent < budget_s / 2 or not times:
            t = smp.step_seconds(threads)
            times.append(t)
            spent += t * len(smp.layers) / cfg.layers + 1e-3
            if len(times) >= 50:
                break
        out[threads] = (float(np.median(times)), len(times))
    step_s, n = out[cores]
    line = {"value": cfg.T / step_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": smp.describe(cores) + f"; median of {n} passes"}
    s1, n1 = out[1]
    line["single_thread"] = {"value": cfg.T / s1, "unit": "tokens/s", "cores": 1, "passes": n1}
    return line


def run_reference(args, world, rank):
    """The reference arm: the fp64 CPU oracle, timed on the host cores."""
    if rank != 0:
        return
    from adapter_pregate_router_b200 import workloads as W
    cfg = W.CONFIGS[args.workload]
    per_step_budget = min(args.ref_budget, 150.0 / (args.steps + args.warmup))
    smp = OracleSample(cfg, layer_budget_s=per_step_budget)
    cores = host_cores()
    for _ in range(args.warmup):
        smp.step_seconds(cores)
    per_step = [smp.step_seconds(cores) for _ in range(args.steps)]
    step_s = float(np.mean(per_step))
    value = cfg.T / step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(cfg, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": smp.describe(cores)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_block(cfg, world):
    full = W_CONFIG_LAYERS.get(cfg.name, cfg.layers)
    descr = DESCR.get(cfg.name, cfg.name)
    if cfg.layers != full:
        descr += f" [REDUCED: {cfg.layers} of {full} layers, profiling only]"
    return {"workload": descr, "name": cfg.name, "tokens_per_step": cfg.T,
            "adapters": cfg.E, "top_k": cfg.k, "ranks": list(cfg.rank_choices), "layers": cfg.layers,
            "parallelism": f"replicas x{world} (token batches, no collective)",
            "l2": ("working set fits in the 126 MB L2 (parity case, no roofline claim)" if cfg.name == "tiny" else
                   "working set larger than the 126 MB L2 (every layer has its own buffers); no flush")}


# ---------------------------------------------------------------- GPU leg

# Pinned host copies of a whole step's activations up to this size; above it (prefill: 35 GB in,
# 22 GB out) one layer's worth of pinned host memory is reused for every layer's copies.
E2E_FULL_PINNED_BYTES = 8 << 30


def _e2e(step, cfg, stream, world, nsteps):
    """End to end through the public API: every step copies its activations in from pinned host
    memory, makes the eager C-ABI calls of the step and copies the outputs back, on one stream,
    timed with CUDA events (max over ranks)."""
    import torch
    act_in, act_out = step.act_in, step.act_out
    el = act_in.element_size()
    layers = step.layers
    lin = [step.layer_in[l] for l in layers]
    lout = [step.layer_out[l] for l in layers]
    head = lin[0][0]                       # router input (and nothing else) before the first layer
    full = (act_in.numel() + act_out.numel()) * el <= E2E_FULL_PINNED_BYTES
    if full:
        host_in = torch.empty(act_in.numel(), dtype=act_in.dtype, pin_memory=True)
        host_out = torch.empty(act_out.numel(), dtype=act_out.dtype, pin_memory=True)
        host_in.copy_(act_in)
        note = "whole step's activations in pinned host memory"
    else:
        n_in, n_out = lin[0][1] - lin[0][0], lout[0][1] - lout[0][0]
        host_in = torch.empty(head + n_in, dtype=act_in.dtype, pin_memory=True)
        host_out = torch.empty(n_out, dtype=act_out.dtype, pin_memory=True)
        host_in[:head].copy_(act_in[:head])
        host_in[head:].copy_(act_in[lin[0][0]:lin[0][1]])
        note = ("one layer's activations in pinned host memory, copied in for every layer (bounds pinned host "
                "memory); every layer's inputs and outputs still cross PCIe each step")
    h2d = d2h = 0

    def one_step():
        nonlocal h2d, d2h
        h2d = d2h = 0
        act_in[:head].copy_(host_in[:head], non_blocking=True)
        h2d += head * el
        step.route()
        if cfg.merge:
            step.merge_all()
        for l, (a0, a1), (b0, b1) in zip(layers, lin, lout):
            src = host_in[a0:a1] if full else host_in[head:]
            act_in[a0:a1].copy_(src, non_blocking=True)
            h2d += (a1 - a0) * el
            step.run_layer(l)
            dst = host_out[b0:b1] if full else host_out
            dst.copy_(act_out[b0:b1], non_blocking=True)
            d2h += (b1 - b0) * el

    with torch.cuda.stream(stream):
        for _ in range(2):
            one_step()
        stream.synchronize()
        barrier(world)
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        x0.record(stream)
        for _ in range(nsteps):
            one_step()
        x1.record(stream)
    stream.synchronize()
    wall = time.perf_counter() - t0
    e_ms = max_over_ranks(x0.elapsed_time(x1), world)
    return {"value": cfg.T * nsteps * world / (e_ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": nsteps,
            "ms_per_step": e_ms / nsteps, "host_wall_ms_per_step": wall * 1e3 / nsteps,
            "calls": "eager C-ABI calls (route, segments, every layer call) on one stream", "host_buffers": note}


def measure(name, args, world, rank, local, peaks, kernel_name="auto"):
    """One full-size workload: launches counted, the step captured in a CUDA graph, K timed
    replays (clocks sampled), the SGMM calls alone timed for the roofline, and the e2e leg."""
    import torch
    from adapter_pregate_router_b200 import apr, pipeline
    from adapter_pregate_router_b200 import workloads as W

    cfg_name, base = BASE_MODE.get(name, (name, None))
    cfg = W.scaled(W.CONFIGS[cfg_name], seed=W.CONFIGS[cfg_name].seed + rank)
    if args.layers:
        cfg = W.scaled(cfg, layers=args.layers)
    dev = torch.device("cuda", local)
    kernels = {"auto": apr.SGMM_AUTO, "skinny": apr.SGMM_SKINNY, "tensor": apr.SGMM_TENSOR,
               "dense": apr.SGMM_DENSE, "bank": apr.SGMM_BANK}
    step = pipeline.Step(cfg, device=dev, kernel=kernels[kernel_name], base=base)
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream(dev))

    # launches per step (eager, counted by the library)
    with torch.cuda.stream(stream):
        before = apr.kernel_launches()
        step.run()
        launches = apr.kernel_launches() - before
    stream.synchronize()
    apr.stream_status(step.ws, stream)

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        step.run()
        stream.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            step.run()
    layer_graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(layer_graph, stream=stream):
            step.layers_only()
    stream.synchronize()

    # ---- warm-up
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graph.replay()
    stream.synchronize()
    apr.stream_status(step.ws, stream)

    # ---- timed region: K whole steps
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            ev1.record(stream)
        stream.synchronize()
    torch.cuda.synchronize(dev)
    barrier(world)
    value, ms = aggregate_throughput(cfg.T * args.steps, ev0.elapsed_time(ev1), world)
    ms_step = ms / args.steps
    apr.stream_status(step.ws, stream)

    # ---- the SGMM (or merge + GEMV) calls alone, every layer, no route
    with torch.cuda.stream(stream):
        for _ in range(3):
            layer_graph.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        nrep = max(5, min(args.steps, 200))
        for _ in range(nrep):
            layer_graph.replay()
        e1.record(stream)
    stream.synchronize()
    layer_ms = max_over_ranks(e0.elapsed_time(e1) / nrep, world)
    idx_np = step.idx.cpu().numpy()
    step_bytes = step.algorithmic_bytes(idx_np)
    el = 2 if cfg.dtype == "bf16" else 4
    router_bytes = cfg.T * cfg.d_router * el + cfg.E * cfg.d_router * el
    layer_bytes = step_bytes - router_bytes
    ncalls = len(step.calls) if not cfg.merge else 1 + step.nmerge
    achieved_gbs = layer_bytes / (layer_ms * 1e-3) / 1e9
    traffic = measured_traffic(name) if not args.layers else None
    roof = {
        "bound": "hbm",
        "kernel": ("apr_merge_adapters_planned + apr_gemv (the merge launch and every weight's GEMV)" if cfg.merge
                   else "apr_sgmm_shrink_expand (shrink + expand launches of every layer call)"),
        "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": achieved_gbs / peaks["hbm_gbs"], "peak_source": f"{peaks['source']} copy bandwidth",
        "traffic": traffic,
        "traffic_source": (f"{TRAFFIC_FILE} (ncu, bytes per call, kernel-source hash {kernel_source_hash()})"
                           if traffic is not None else "no capture at the current kernel sources"),
        "bytes_per_call": layer_bytes / ncalls, "calls_per_step": ncalls,
        "us_per_call": layer_ms * 1e3 / ncalls, "step_bytes": step_bytes,
        "step_frac": step_bytes / (ms_step * 1e-3) / 1e9 / peaks["hbm_gbs"],
    }
    if base is not None:
        # base projections and adapters: a contraction, bounded by the tensor cores
        flops = step.flops()
        tflops = flops / (layer_ms * 1e-3) / 1e12
        roof = {
            "bound": "tensor",
            "kernel": "apr_linear_lora (shrink, pack and the fused GEMM of every layer call)",
            "achieved": tflops, "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
            "frac": tflops / peaks["bf16_tflops_sustained"],
            "peak_source": f"{peaks['source']} sustained bf16 dense (a long step under the power cap)",
            "traffic": traffic,
            "traffic_source": (f"{TRAFFIC_FILE} (ncu, bytes per call, kernel-source hash {kernel_source_hash()})"
                               if traffic is not None else "no capture at the current kernel sources"),
            "flops_per_step": flops, "calls_per_step": ncalls, "us_per_call": layer_ms * 1e3 / ncalls,
            "hbm_frac": layer_bytes / (layer_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "step_bytes": step_bytes,
        }
    graph.reset()
    layer_graph.reset()
    e2e = _e2e(step, cfg, stream, world, max(3, min(args.steps, 20 if cfg.T < 4096 else 3)))
    apr.stream_status(step.ws, stream)
    out = {"cfg": cfg, "value": value, "ms_per_step": ms_step, "roofline": roof, "e2e": e2e,
           "clocks": clk.summary(), "gpu_launches": launches * args.steps, "launches_per_step": launches,
           "config": dict(config_block(cfg, world), **({"sgmm_kernel": kernel_name} if kernel_name != "auto" else {}),
                          **({"base": base} if base else {}))}
    del step
    import gc
    gc.collect()
    torch.cuda.empty_cache()
    if base == "fused":
        # the pipeline the fused call replaces: a library GEMM into y, then the SGMM call adding the
        # adapters in place, same layers, weights and routing, timed the same way (layer calls only)
        ref = pipeline.Step(cfg, device=dev, base="cublas")
        with torch.cuda.stream(stream):
            ref.route()
            ref.layers_only()
            stream.synchronize()
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2, stream=stream):
                ref.layers_only()
            for _ in range(3):
                g2.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(nrep):
                g2.replay()
            e1.record(stream)
        stream.synchronize()
        apr.stream_status(ref.ws, stream)
        un_ms = max_over_ranks(e0.elapsed_time(e1) / nrep, world)
        out["unfused"] = {"layers_ms": un_ms, "fused_layers_ms": layer_ms, "speedup": un_ms / layer_ms,
                          "pipeline": "torch.matmul base GEMM into y, then apr_sgmm_shrink_expand in place (auto)"}
        g2.reset()
        del ref
        gc.collect()
        torch.cuda.empty_cache()
    return out


def merge_crossover(args, world, rank, local, batches=(1, 2, 4, 8)):
    """Merge in place vs unmerged adapters for a batch of T tokens that share one routing
    (the 224 decode-shaped weights of the merge workload, its first token's top-2 adapters).
    Per step, merged: a library GEMM of the T rows on every merged weight; unmerged: the same
    GEMM on W plus the SGMM call of every (layer, group) adding the adapters.  The in-place
    merge + exact unmerge is paid once per routing change, so merging pays after
    N* = (merge + unmerge) / (unmerged - merged) steps with the same adapters."""
    import torch
    from adapter_pregate_router_b200 import apr
    from adapter_pregate_router_b200 import workloads as W

    cfg = W.scaled(W.CONFIGS["merge"], seed=W.CONFIGS["merge"].seed + rank)
    if args.layers:
        cfg = W.scaled(cfg, layers=args.layers)
    dev = torch.device("cuda", local)
    E, k, r = cfg.E, cfg.k, 16
    Tmax = max(batches)
    h, Wr, _ = W.router_inputs(cfg)
    ws = apr.workspace(Tmax, k, E, r, max(g.d_in for g in cfg.groups), device=dev)
    idx1 = torch.empty((1, k), dtype=torch.int32, device=dev)
    gate1 = torch.empty((1, k), dtype=torch.float32, device=dev)
    apr.pregate_route(torch.from_numpy(h).to(dev, torch.bfloat16), torch.from_numpy(Wr).to(dev, torch.bfloat16),
                      k, idx1, gate1, ws)
    ranks = torch.full((E,), r, dtype=torch.int32, device=dev)
    entries, groups, keep = [], [], []
    for l in range(cfg.layers):
        for g in cfg.groups:
            x = W.device_tensor(cfg, W.xm_key(l, g.name, g.proj_names[0]), (Tmax * g.d_in,), dev).view(Tmax, g.d_in)
            projs = []
            for p, d_out in zip(g.proj_names, g.d_outs):
                Wt = W.device_tensor(cfg, W.w_key(l, g.name, p), (d_out, g.d_in), dev)
                A = [W.device_tensor(cfg, W.a_key(l, g.name, p, e), (r, g.d_in), dev) for e in range(E)]
                B = [W.device_tensor(cfg, W.b_key(l, g.name, p, e), (d_out, r), dev) for e in range(E)]
                At, Bt = apr.ptr_array(A, dev), apr.ptr_array(B, dev)
                R = apr.merge_residual(Wt)
                y = torch.empty((Tmax, d_out), dtype=torch.bfloat16, device=dev)
                entries.append((Wt, R, At, Bt))
                projs.append((Wt, y, At, Bt))
                keep += [A, B]
            groups.append((x, projs))
    W.clear_device_pools()
    nmerge = len(entries)
    table = apr.merge_table(entries, dev)
    esc = apr.merge_escapes(1 << 22, dev)
    stream = torch.cuda.Stream(device=dev)

    def timed(fn, reps):
        with torch.cuda.stream(stream):
            fn()
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn()
            for _ in range(2):
                g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        stream.synchronize()
        apr.stream_status(ws, stream)
        g.reset()
        return max_over_ranks(e0.elapsed_time(e1) / reps, world)

    def merge_unmerge():
        apr.merge_adapters_inplace(table, nmerge, E, r, idx1, gate1, k, esc, ws)
        apr.unmerge_adapters_inplace(table, nmerge, E, r, idx1, gate1, k, esc, ws)

    mu_ms = timed(merge_unmerge, 5)
    rows = []
    for T in batches:
        idx = idx1.expand(T, k).contiguous()
        gate = gate1.expand(T, k).contiguous()
        seg_off = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(T * k, dtype=torch.int32, device=dev)
        apr.segment_tokens(idx, E, seg_off, perm, ws)
        calls = []
        for x, projs in groups:
            xt = x[:T]
            pj = [apr.make_proj(y[:T], y[:T], At, Bt) for (_, y, At, Bt) in projs]
            calls.append((xt, [(Wt, y[:T]) for (Wt, y, _, _) in projs], pj))

        def base_only():
            for xt, gemms, _ in calls:
                for Wt, yt in gemms:
                    torch.matmul(xt, Wt.t(), out=yt)

        def unmerged():
            for xt, gemms, pj in calls:
                for Wt, yt in gemms:
                    torch.matmul(xt, Wt.t(), out=yt)
                apr.sgmm_shrink_expand(xt, pj, k, E, ranks, r, idx, gate, seg_off, perm, ws)

        m_ms = timed(base_only, 10)
        u_ms = timed(unmerged, 10)
        extra = u_ms - m_ms
        rows.append({"T": T, "merged_step_ms": m_ms, "unmerged_step_ms": u_ms,
                     "steps_to_pay_back": (mu_ms / extra) if extra > 0 else None})
    del table, entries, groups, keep
    import gc
    gc.collect()
    torch.cuda.empty_cache()
    return {"weights": nmerge, "merge_plus_unmerge_ms": mu_ms,
            "merged": "in-place merge, library GEMM of the T rows on W', exact in-place unmerge",
            "unmerged": "library GEMM on W, then apr_sgmm_shrink_expand per (layer, group) in place",
            "batches": rows}


def run_gpu(args, world, rank, local):
    from adapter_pregate_router_b200 import workloads as W
    peaks = load_peaks()
    main = measure(args.workload, args, world, rank, local, peaks, args.kernel)
    cfg = main["cfg"]
    others = {}
    also = [] if args.also in ("", "none") else [w.strip() for w in args.also.split(",")]
    for name in also:
        if name == args.workload:
            continue
        if name == "merge_crossover":
            others[name] = merge_crossover(args, world, rank, local)
            continue
        r = measure(name, args, world, rank, local, peaks)
        others[name] = {"value": r["value"], "unit": "tokens/s", "ms_per_step": r["ms_per_step"],
                        "config": r["config"], "roofline": r["roofline"], "e2e": r["e2e"], "clocks": r["clocks"],
                        "gpu_launches": r["gpu_launches"], "launches_per_step": r["launches_per_step"]}
        if "unfused" in r:
            others[name]["unfused"] = r["unfused"]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(W.CONFIGS[BASE_MODE.get(args.workload, (args.workload,))[0]], budget_s=args.ref_budget)

    line = {
        "metric": METRIC, "value": main["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": main["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if cfg.dtype == "bf16" else "f32", "data": "synthetic",
        "config": main["config"], "roofline": main["roofline"], "cpu_baseline": cpu, "e2e": main["e2e"],
        "clocks": main["clocks"], "gpu_launches": main["gpu_launches"],
        "launches_per_step": main["launches_per_step"],
    }
    if "unfused" in main:
        line["unfused"] = main["unfused"]
    if others:
        line["workloads"] = others
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill",
                    choices=["decode", "prefill", "multitenant", "merge", "tiny", "prefill_fused"])
    ap.add_argument("--also", default="decode,multitenant,merge,prefill_fused,merge_crossover",
                    help="other full-size workloads timed in the same run and reported under 'workloads' "
                         "(comma-separated, or 'none')")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-budget", type=float, default=12.0, help="seconds of oracle work per reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", default="auto", choices=["auto", "skinny", "tensor", "dense", "bank"],
                    help="force one SGMM kernel class on the main workload (comparisons; the benchmark uses auto)")
    ap.add_argument("--layers", type=int, default=0,
                    help="build only this many layers (a reduced workload for profiling; not the benchmark)")
    ap.add_argument("--ingest-traffic", metavar="CSV",
                    help="record an ncu DRAM capture of --workload as bytes per call (with --calls, --command)")
    ap.add_argument("--calls", type=float, default=1.0)
    ap.add_argument("--command", default="")
    ap.add_argument("--kernels", default=None, help="regex of the kernel names to ingest")
    ap.add_argument("--last", type=int, default=0, help="ingest only the last N matching launches")
    args = ap.parse_args()
    if args.ingest_traffic:
        print(ingest_traffic(args.ingest_traffic, args.workload, args.calls, args.command, args.kernels, args.last))
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args)
    try:
        run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
