"""Throughput of the fused attention forward + backward step on B200 (sm_100a).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one pass of the whole hot path over one batch: fa_fwd (O, LSE) -- or, on the
workloads whose heads are too few to fill the GPU, fa_fwd_splitkv (split forward + LSE
merge) -- followed by fa_bwd (row preprocess, fused main backward kernel, dQ conversion).  Inputs are seeded
synthetic bf16 N(0, 1) tensors of the workload's shape (no dataset exists for this
kernel); FLOPs follow the workload convention: 4*B*H*N^2*d forward, 2.5x that backward,
halved for causal masking.

Multi-GPU (torchrun, one process per GPU): heads are independent, so each rank runs its
own batch of the workload with no data-path collective (weak scaling); the only
communication is the barrier and the max-over-ranks of the device time.

Modes (same JSON line, mode named in ``config``): ``--deterministic`` (int64 fixed-point dQ
accumulation), ``--dropout P`` (fused dropout in both passes), ``--fwd-splits S`` (split-KV
forward), ``--fp8`` (the FP8 E4M3 forward alone, d = 128).

Prints one JSON line on rank 0.  ``--impl reference`` times the fp64 CPU oracle (the only
other implementation of this computation available here) on a bounded sample of the same
workload, on the host cores.
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

METRIC = "attention fwd / fwd+bwd TFLOP/s and % of B200 dense BF16 peak"
DEFAULT_WORKLOAD = "gpt2_B64_H16_N1024_d64"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha(name: str) -> str:
    """Hash of the source file a kernel is built from (ties stored ncu traffic to a version)."""
    src = {"fwd": "fa_fwd.cu", "bwd_main": "fa_bwd.cu"}[name]
    files = [os.path.join(ROOT, "exact_attention_111_b200", "csrc", f) for f in (src, "sm100.cuh", "fa_internal.h")]
    h = hashlib.sha256()
    for f in files:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel, {}).get(workload)
    if not e or e.get("source_sha") != kernel_source_sha(kernel):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank device time over all ranks (NCCL on GPUs, gloo in CPU tests)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch of heads (weak scaling over independent heads)."""
    return base_seed + 7919 * rank


def aggregate_tflops(world: int, flops_per_rank_step: float, steps: int, max_elapsed_ms: float) -> float:
    """Whole-job throughput: the work of all ranks over the slowest rank's device time."""
    return world * flops_per_rank_step * steps / (max_elapsed_ms * 1e-3) / 1e12


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("internal_api") in ("openblas", "mkl", "blis")]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def oracle_sample(w, seconds: float, max_heads: int | None = None):
    """Time the fp64 oracle (forward + backward, whole heads) on host cores for about
    ``seconds``; returns (heads done, elapsed s, FLOPs by the workload convention)."""
    import numpy as np
    import oracle.attention as ora
    from exact_attention_111_b200.inputs import attention_flops, butterfly_blockmask, make_inputs
    inp = make_inputs(1, 1, w.N, w.d, w.seed, k_scale=w.k_scale)
    q, k, v, do = (inp[n][0, 0].double().numpy() for n in ("q", "k", "v", "dout"))
    mask = butterfly_blockmask(w.tiles).numpy() if w.butterfly else None
    t0 = time.perf_counter()
    heads = 0
    while True:
        ora.attention_bwd_head(q, k, v, do, w.scale, w.causal, mask)
        heads += 1
        el = time.perf_counter() - t0
        if (seconds > 0 and el >= seconds) or (max_heads and heads >= max_heads):
            break
    flops = heads * attention_flops(1, 1, w.N, w.d, w.causal, True)
    return heads, el, flops


def run_reference(args, w, world, rank):
    """fp64 CPU oracle on the host cores: a bounded sample of heads per step."""
    if rank != 0:
        return
    from exact_attention_111_b200.inputs import attention_flops
    per_head = attention_flops(1, 1, w.N, w.d, w.causal, True)
    # heads per step sized so the whole run stays within a few minutes
    _, t1, _ = oracle_sample(w, 0.0, max_heads=1)
    budget = 120.0 / max(1, args.steps + args.warmup)
    hps = max(1, int(budget / max(t1, 1e-6)))
    for _ in range(args.warmup):
        oracle_sample(w, 0.0, max_heads=hps)
    times = []
    for _ in range(args.steps):
        _, el, _ = oracle_sample(w, 0.0, max_heads=hps)
        times.append(el)
    tot = sum(times)
    value = args.steps * hps * per_head / tot / 1e12
    sample = f"{hps} whole (b, h) heads of {w.name} per step (forward + backward, fp64 numpy/BLAS)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, world):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "blockmask": "butterfly+global first row/col" if w.butterfly else None,
            "k_scale": w.k_scale, "per_rank": "each rank runs its own batch of B*H heads",
            "parallelism": f"replicas x{world} (heads independent, no collective)"}


def run_ours(args, w, world, rank, local):
    import torch
    import exact_attention_111_b200 as fa
    from exact_attention_111_b200.inputs import attention_flops, butterfly_blockmask, make_inputs

    fa.lib()  # fails loudly when the CUDA library is missing
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    inp = make_inputs(w.B, w.H, w.N, w.d, rank_seed(w.seed, rank), k_scale=w.k_scale)
    host = {n: inp[n].pin_memory() for n in ("q", "k", "v", "dout")}
    d = {n: t.to(dev) for n, t in host.items()}
    mask = butterfly_blockmask(w.tiles).to(dev) if w.butterfly else None
    B, H, N, D = w.B, w.H, w.N, w.d
    scale = w.scale
    o = torch.empty_like(d["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"])
    det = bool(args.deterministic)
    wsb = fa.fa_bwd_workspace_bytes_ex(B, H, N, D, det)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    splits = None
    if w.fwd_splits is not None:
        splits = w.fwd_splits or fa.fa_splitkv_choose(B, H, N, w.causal,
                                                      torch.cuda.get_device_properties(dev).multi_processor_count)
        wsfb = fa.fa_fwd_splitkv_workspace_bytes(B, H, N, D, splits)
        wsf = torch.empty(wsfb, dtype=torch.uint8, device=dev)

    pdrop, dseed = float(args.dropout), 0x5EED
    if pdrop > 0 and splits is not None:
        raise SystemExit("--dropout does not combine with the split-KV forward")

    def forward(q, k, v, o_, lse_):
        if pdrop > 0:
            fa.fa_fwd_ex(q, k, v, o_, lse_, B, H, N, D, scale, w.causal, mask, fa.FA_BF16, False, None, stream,
                         dropout_p=pdrop, dropout_seed=dseed)
        elif splits is None:
            fa.fa_fwd(q, k, v, o_, lse_, B, H, N, D, scale, w.causal, mask, stream)
        else:
            fa.fa_fwd_splitkv(q, k, v, o_, lse_, B, H, N, D, scale, w.causal, mask, splits, wsf, wsfb, stream)
    in_bytes = sum(t.numel() * t.element_size() for t in d.values())

    ev_f = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

    launches = [0]

    def step(timed_kernels=None):
        if timed_kernels is not None:
            timed_kernels["f0"].record(stream)
        forward(d["q"], d["k"], d["v"], o, lse)
        launches[0] += fa.fa_last_launch_count()
        if timed_kernels is not None:
            timed_kernels["f1"].record(stream)
        fa.fa_bwd_ex(d["q"], d["k"], d["v"], o, lse, d["dout"], dq, dk, dv, B, H, N, D, scale, w.causal, mask,
                     fa.FA_BF16, None, ws, wsb, stream,
                     timed_kernels["b0"] if timed_kernels else None, timed_kernels["b1"] if timed_kernels else None,
                     deterministic=det, dropout_p=pdrop, dropout_seed=dseed)
        launches[0] += fa.fa_last_launch_count()

    # ---------------------------------------------------------------- warm-up
    for _ in range(args.warmup):
        step()
    fa.fa_check_status(stream)

    # ---------------------------------------------------------------- timed region
    per_kernel = {"fwd": [], "bwd_main": []}
    kev = [{"f0": torch.cuda.Event(enable_timing=True), "f1": torch.cuda.Event(enable_timing=True),
            "b0": torch.cuda.Event(enable_timing=True), "b1": torch.cuda.Event(enable_timing=True)}
           for _ in range(args.steps)]
    for e in kev:  # torch creates the CUDA event lazily: record once so the library gets a handle
        for ev in e.values():
            ev.record(stream)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(world)
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.25)
    launches[0] = 0
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        step(kev[i])
    stop.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    barrier(world)
    fa.fa_check_status(stream)
    gpu_launches = launches[0]
    elapsed_ms = start.elapsed_time(stop)
    for e in kev:
        per_kernel["fwd"].append(e["f0"].elapsed_time(e["f1"]))
        per_kernel["bwd_main"].append(e["b0"].elapsed_time(e["b1"]))
    elapsed_ms = max_over_ranks(elapsed_ms, world)

    fwd_flops = attention_flops(B, H, N, D, w.causal, False)
    step_flops = attention_flops(B, H, N, D, w.causal, True)
    bwd_flops = step_flops - fwd_flops
    ms_step = elapsed_ms / args.steps
    value = aggregate_tflops(world, step_flops, args.steps, elapsed_ms)
    fwd_ms = statistics.mean(per_kernel["fwd"])
    bmain_ms = statistics.mean(per_kernel["bwd_main"])
    fwd_tflops = fwd_flops / (fwd_ms * 1e-3) / 1e12
    bmain_tflops = bwd_flops / (bmain_ms * 1e-3) / 1e12

    # ---------------------------------------------------------------- end to end (host buffers)
    # Every step copies its inputs from pinned host memory and its results (O, LSE, dQ, dK, dV)
    # back to pinned host memory.  Device buffers are double-buffered and three streams
    # (host->device, compute, device->host) overlap step k+1's upload and step k-1's download
    # with step k's kernels; the timed region spans the first upload to the last download.
    e2e_steps = max(3, min(args.steps, 20))
    sets = []
    for _ in range(2):
        din = {n: torch.empty_like(t) for n, t in d.items()}
        dout_ = {"o": torch.empty_like(o), "lse": torch.empty_like(lse), "dq": torch.empty_like(dq),
                 "dk": torch.empty_like(dk), "dv": torch.empty_like(dv)}
        sets.append((din, dout_))
    host_out = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in sets[0][1].items()}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(nsteps, t0=None, t1=None):
        if t0 is not None:
            t0.record(s_up)
        for k in range(nsteps):
            b = k % 2
            din, dres = sets[b]
            if k >= 2:
                s_up.wait_event(ev_comp[b])          # step k-2 finished reading these inputs
            with torch.cuda.stream(s_up):
                for n in host:
                    din[n].copy_(host[n], non_blocking=True)
            ev_up[b].record(s_up)
            stream.wait_event(ev_up[b])
            if k >= 2:
                stream.wait_event(ev_down[b])        # step k-2's results are on the host
            forward(din["q"], din["k"], din["v"], dres["o"], dres["lse"])
            fa.fa_bwd_ex(din["q"], din["k"], din["v"], dres["o"], dres["lse"], din["dout"], dres["dq"], dres["dk"],
                         dres["dv"], B, H, N, D, scale, w.causal, mask, fa.FA_BF16, None, ws, wsb, stream,
                         deterministic=det, dropout_p=pdrop, dropout_seed=dseed)
            ev_comp[b].record(stream)
            s_down.wait_event(ev_comp[b])
            with torch.cuda.stream(s_down):
                for n, t in dres.items():
                    host_out[n].copy_(t, non_blocking=True)
            ev_down[b].record(s_down)
        if t1 is not None:
            s_down.wait_stream(s_up)
            s_down.wait_stream(stream)
            t1.record(s_down)

    e2e_run(2)
    torch.cuda.synchronize(dev)
    barrier(world)
    s2, t2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(e2e_steps, s2, t2)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(s2.elapsed_time(t2), world)
    e2e_value = aggregate_tflops(world, step_flops, e2e_steps, e2e_ms)
    fa.fa_check_status(stream)

    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    peak_burst = float(peaks["bf16_tflops"])
    peak_sust = float(peaks.get("bf16_tflops_sustained", peak_burst))
    # dominant kernel: the one with the larger share of the step time
    if bmain_ms >= fwd_ms:
        dom, dom_tf, dom_flops = "bwd_main", bmain_tflops, bwd_flops
    else:
        dom, dom_tf, dom_flops = "fwd", fwd_tflops, fwd_flops
    traffic = stored_traffic(dom, w.name) if not (det or pdrop > 0) else None   # captured for the default mode only
    roofline = {"bound": "tensor", "achieved": dom_tf, "peak": peak_sust, "unit": "TFLOP/s",
                "frac": dom_tf / peak_sust, "traffic": traffic, "kernel": dom,
                "peak_source": f"bf16_tflops_sustained of {peak_src} (MEASURED_PEAKS.json)",
                "frac_of_burst_peak": dom_tf / peak_burst,
                "algorithmic_flops_per_launch": dom_flops}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w, world),
                       **({"fwd_splits": splits, "fwd": "fa_fwd_splitkv (split forward + LSE merge, "
                           "both inside the fwd timing)"} if splits is not None else {}),
                       **({"deterministic_bwd": "int64 fixed-point dQ accumulation"} if det else {}),
                       **({"dropout_p": pdrop, "dropout": "fused, Philox4x32-10 mask regenerated in the backward"}
                          if pdrop > 0 else {}),
                       l2=f"inputs {in_bytes / 2**20:.0f} MiB per rank > 126 MiB L2, no flush"
                       if in_bytes > L2_BYTES else "inputs fit in L2"),
        "fwd_tflops": fwd_tflops, "fwd_ms": fwd_ms, "bwd_main_tflops": bmain_tflops, "bwd_main_ms": bmain_ms,
        "fwd_bwd_frac_of_peak": value / world / peak_burst, "fwd_frac_of_peak": fwd_tflops / peak_burst,
        "peak_bf16_tflops_burst": peak_burst,
        "roofline": roofline,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps},
        "gpu_launches": gpu_launches,
        "clocks": clocks,
    }
    if not args.no_cpu_baseline and world == 1:
        heads, el, flops = oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
                                "kind": "oracle",
                                "sample": f"{heads} whole (b, h) heads of {w.name}, forward + backward, "
                                          f"{el:.1f} s, fp64 numpy/BLAS"}
    print(json.dumps(line), flush=True)


def run_fp8(args, w, world, rank, local):
    """FP8 (E4M3) forward alone: one step = the V transpose + the fused forward over one batch
    of the workload, quantized per tensor (there is no FP8 backward)."""
    import torch
    import exact_attention_111_b200 as fa
    from exact_attention_111_b200.inputs import attention_flops, butterfly_blockmask, make_inputs, quantize_e4m3

    fa.lib()
    if w.d != 128:
        raise SystemExit("--fp8 needs a d = 128 workload")
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    inp = make_inputs(w.B, w.H, w.N, w.d, rank_seed(w.seed, rank), k_scale=w.k_scale, with_dout=False)
    qz = {n: quantize_e4m3(inp[n]) for n in ("q", "k", "v")}
    host = {n: qz[n][0].view(torch.uint8).pin_memory() for n in qz}
    d8 = {n: t.to(dev) for n, t in host.items()}
    ds = {n: qz[n][1] for n in qz}
    mask = butterfly_blockmask(w.tiles).to(dev) if w.butterfly else None
    B, H, N, D = w.B, w.H, w.N, w.d
    o = torch.empty((B, H, N, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    wsb = fa.fa_fwd_fp8_workspace_bytes(B, H, N, D)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(src):
        fa.fa_fwd_fp8(src["q"], src["k"], src["v"], ds["q"], ds["k"], ds["v"], o, lse, B, H, N, D, w.scale, w.causal,
                      mask, False, ws, wsb, stream)

    for _ in range(args.warmup):
        step(d8)
    fa.fa_check_status(stream)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(world)
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.25)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        step(d8)
    stop.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    barrier(world)
    fa.fa_check_status(stream)
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), world)
    flops = attention_flops(B, H, N, D, w.causal, False)
    value = aggregate_tflops(world, flops, args.steps, elapsed_ms)
    # end to end: E4M3 codes up from pinned host memory, O and LSE back, every step
    host_o = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    host_l = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    e2e_steps = max(3, min(args.steps, 20))
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    s0.record(stream)
    for _ in range(e2e_steps):
        for n in d8:
            d8[n].copy_(host[n], non_blocking=True)
        step(d8)
        host_o.copy_(o, non_blocking=True)
        host_l.copy_(lse, non_blocking=True)
    s1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(s0.elapsed_time(s1), world)
    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    peak8 = 2.0 * float(peaks["bf16_tflops"])
    tf = value / world
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": dict(workload_config(w, world), mode="fp8 forward only (E4M3 Q, K, V with per-tensor "
                                                      "dequantisation; V transpose + fused forward per step)"),
        "roofline": {"bound": "tensor", "achieved": tf, "peak": peak8, "unit": "TFLOP/s", "frac": tf / peak8,
                     "traffic": None, "kernel": "fwd_fp8 (+ vt transpose)",
                     "peak_source": f"2 x bf16_tflops of {peak_src} (MEASURED_PEAKS.json x nominal fp8/bf16 ratio)"},
        "e2e": {"value": aggregate_tflops(world, flops, e2e_steps, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": sum(t.numel() for t in host.values()),
                "d2h_bytes_per_step": host_o.numel() * 2 + host_l.numel() * 4, "steps": e2e_steps},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fwd-splits", type=int, default=None,
                    help="forward through fa_fwd_splitkv with this many key ranges (0: chosen for the "
                         "GPU; default: the workload's own setting)")
    ap.add_argument("--dropout", type=float, default=0.0,
                    help="fused dropout probability in both passes (default 0: none)")
    ap.add_argument("--fp8", action="store_true",
                    help="time the FP8 (E4M3) forward alone on the workload (d = 128)")
    ap.add_argument("--deterministic", action="store_true",
                    help="backward in deterministic mode (bitwise repeatable dQ)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from exact_attention_111_b200.inputs import workloads
    w = workloads()[args.workload]
    if args.fwd_splits is not None:
        import dataclasses
        w = dataclasses.replace(w, fwd_splits=args.fwd_splits)
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, w, world, rank)
        return
    world, rank, local = dist_setup()
    try:
        (run_fp8 if args.fp8 else run_ours)(args, w, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
