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
# The largest single-GPU workload: one batch of 32 heads of 16384 tokens at d = 128, causal,
# with K scaled by 4 (peaked softmax rows).
DEFAULT_WORKLOAD = "long_B1_H32_N16384_d128_causal_k4"
# The d = 128, N >= 4k non-causal regime the throughput targets are stated for, timed in the
# same run and reported beside the main line.
TARGET_POINT = "sweep_B1_H16_N16384_d128"
# Peaks measured on this machine's B200s when MEASURED_PEAKS.json is absent: a STREAM-style copy
# and a cuBLAS bf16 GEMM as a burst (1590) and as a seconds-long loop under the 1000 W power
# cap, where it settles near 1400 at about 1.3 GHz.
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's B200 dense BF16 tensor rating: the HGX B200 sheet gives 36 PFLOP/s per 8 GPUs with
# 2:4 sparsity, i.e. 2.25 PFLOP/s dense per GPU.
NOMINAL_DENSE_BF16_TFLOPS = 2250.0
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


def oracle_sample(w, seconds: float, max_heads: int | None = None, n_tokens: int | None = None):
    """Time the fp64 oracle (forward + backward of one head at a time) on host cores for about
    ``seconds`` (or ``max_heads`` heads); returns (heads done, elapsed s, FLOPs by the workload
    convention).  ``n_tokens`` < N runs each head over its first n_tokens tokens only (queries
    and keys): a smaller problem of the same kind, for sequences whose whole head takes the
    oracle too long."""
    import numpy as np
    import oracle.attention as ora
    from exact_attention_111_b200.inputs import attention_flops, butterfly_blockmask, make_inputs
    n = w.N if n_tokens is None else min(n_tokens, w.N)
    inp = make_inputs(1, 1, w.N, w.d, w.seed, k_scale=w.k_scale)
    q, k, v, do = (inp[x][0, 0, :n].double().numpy() for x in ("q", "k", "v", "dout"))
    mask = butterfly_blockmask((n + 127) // 128).numpy() if w.butterfly else None
    t0 = time.perf_counter()
    heads = 0
    while True:
        ora.attention_bwd_head(q, k, v, do, w.scale, w.causal, mask)
        heads += 1
        el = time.perf_counter() - t0
        if (seconds > 0 and el >= seconds) or (max_heads and heads >= max_heads):
            break
    flops = heads * attention_flops(1, 1, n, w.d, w.causal, True)
    return heads, el, flops


def run_reference(args, w, world, rank):
    """fp64 CPU oracle on the host cores: a bounded sample of the workload per step, sized so
    the whole --steps/--warmup run takes about two minutes.  Whole heads when one fits the
    per-step budget; otherwise each step runs one head over its first n tokens, n the largest
    multiple of 128 whose oracle time (quadratic in n) fits."""
    if rank != 0:
        return
    _, t1, _ = oracle_sample(w, 0.0, max_heads=1)
    budget = 120.0 / max(1, args.steps + args.warmup)
    n_tok = w.N
    if t1 > budget:
        n_tok = max(128, int(w.N * math.sqrt(budget / t1)) // 128 * 128)
        hps = 1
    else:
        hps = max(1, int(budget / max(t1, 1e-6)))
    for _ in range(args.warmup):
        oracle_sample(w, 0.0, max_heads=hps, n_tokens=n_tok)
    times, flops = [], 0.0
    for _ in range(args.steps):
        _, el, f = oracle_sample(w, 0.0, max_heads=hps, n_tokens=n_tok)
        times.append(el)
        flops += f
    tot = sum(times)
    value = flops / tot / 1e12
    if n_tok == w.N:
        sample = f"{hps} whole (b, h) heads of {w.name} per step (forward + backward, fp64 numpy/BLAS)"
    else:
        sample = (f"1 (b, h) head of {w.name} over its first {n_tok} of {w.N} tokens per step (forward + "
                  f"backward, fp64 numpy/BLAS; a whole head took {t1:.1f} s)")
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


def input_bytes(w) -> int:
    """Bytes of the step's inputs on one rank: q, k, v, dO (16-bit)."""
    return 4 * w.B * w.H * w.N * w.d * 2


def l2_note(w) -> str:
    b = input_bytes(w)
    return (f"inputs {b / 2**20:.0f} MiB per rank > 126 MiB L2, no flush" if b > L2_BYTES
            else "inputs fit in L2")


def workload_config(w, world):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "blockmask": "butterfly+global first row/col" if w.butterfly else None,
            "k_scale": w.k_scale, "per_rank": "each rank runs its own batch of B*H heads",
            "parallelism": f"replicas x{world} (heads independent, no collective)",
            "l2": l2_note(w)}


class StepSetup:
    """Device buffers, workspace and the launch of one fwd + bwd step for workload ``w``."""

    def __init__(self, args, w, rank, dev):
        import torch
        import exact_attention_111_b200 as fa
        from exact_attention_111_b200.inputs import butterfly_blockmask, make_inputs

        self.fa, self.w, self.dev = fa, w, dev
        inp = make_inputs(w.B, w.H, w.N, w.d, rank_seed(w.seed, rank), k_scale=w.k_scale)
        self.host = {n: inp[n].pin_memory() for n in ("q", "k", "v", "dout")}
        self.d = {n: t.to(dev) for n, t in self.host.items()}
        self.mask = butterfly_blockmask(w.tiles).to(dev) if w.butterfly else None
        B, H, N, D = w.B, w.H, w.N, w.d
        self.o = torch.empty_like(self.d["q"])
        self.lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        self.dq, self.dk, self.dv = (torch.empty_like(self.d[n]) for n in ("q", "k", "v"))
        self.det = bool(args.deterministic)
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        # the workloads whose heads are too few to fill the GPU also split the backward's query
        # ranges (not combinable with the deterministic mode)
        self.qsplits = (fa.fa_bwd_splitq_choose(B, H, N, w.causal, sms)
                        if w.fwd_splits is not None and not self.det else 0)
        if args.bwd_splits is not None:
            self.qsplits = args.bwd_splits
        self.wsb = (fa.fa_bwd_workspace_bytes_split(B, H, N, D, self.qsplits) if self.qsplits > 1
                    else fa.fa_bwd_workspace_bytes_ex(B, H, N, D, self.det))
        self.ws = torch.empty(self.wsb, dtype=torch.uint8, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        self.splits = None
        if w.fwd_splits is not None:
            self.splits = w.fwd_splits or fa.fa_splitkv_choose(B, H, N, w.causal, sms)
            self.wsfb = fa.fa_fwd_splitkv_workspace_bytes(B, H, N, D, self.splits)
            self.wsf = torch.empty(self.wsfb, dtype=torch.uint8, device=dev)
        self.pdrop, self.dseed = float(args.dropout), 0x5EED
        if self.pdrop > 0 and self.splits is not None:
            raise SystemExit("--dropout does not combine with the split-KV forward")
        self.launches = 0

    def forward(self, q, k, v, o_, lse_):
        fa, w = self.fa, self.w
        B, H, N, D = w.B, w.H, w.N, w.d
        if self.pdrop > 0:
            fa.fa_fwd_ex(q, k, v, o_, lse_, B, H, N, D, w.scale, w.causal, self.mask, fa.FA_BF16, False, None,
                         self.stream, dropout_p=self.pdrop, dropout_seed=self.dseed)
        elif self.splits is None:
            fa.fa_fwd(q, k, v, o_, lse_, B, H, N, D, w.scale, w.causal, self.mask, self.stream)
        else:
            fa.fa_fwd_splitkv(q, k, v, o_, lse_, B, H, N, D, w.scale, w.causal, self.mask, self.splits, self.wsf,
                              self.wsfb, self.stream)
        self.launches += fa.fa_last_launch_count()

    def backward(self, q, k, v, o_, lse_, do_, dq_, dk_, dv_, ev0=None, ev1=None):
        fa, w = self.fa, self.w
        fa.fa_bwd_ex(q, k, v, o_, lse_, do_, dq_, dk_, dv_, w.B, w.H, w.N, w.d, w.scale, w.causal, self.mask,
                     fa.FA_BF16, None, self.ws, self.wsb, self.stream, ev0, ev1,
                     deterministic=self.det, dropout_p=self.pdrop, dropout_seed=self.dseed,
                     query_splits=self.qsplits)
        self.launches += fa.fa_last_launch_count()

    def step(self, ev=None):
        d = self.d
        if ev is not None:
            ev["f0"].record(self.stream)
        self.forward(d["q"], d["k"], d["v"], self.o, self.lse)
        if ev is not None:
            ev["f1"].record(self.stream)
        self.backward(d["q"], d["k"], d["v"], self.o, self.lse, d["dout"], self.dq, self.dk, self.dv,
                      ev["b0"] if ev else None, ev["b1"] if ev else None)


def time_device(st: "StepSetup", steps: int, warmup: int, world: int, sample_clocks: bool):
    """W untimed steps, then K steps bracketed by a barrier and synchronisation; CUDA events on
    the launching stream time the whole region and, per step, the forward and the fused main
    backward kernel.  Returns the times (the region's as the max over ranks)."""
    import torch
    fa, dev, stream = st.fa, st.dev, st.stream
    for _ in range(warmup):
        st.step()
    fa.fa_check_status(stream)
    kev = [{n: torch.cuda.Event(enable_timing=True) for n in ("f0", "f1", "b0", "b1")} for _ in range(steps)]
    for e in kev:  # torch creates the CUDA event lazily: record once so the library gets a handle
        for ev in e.values():
            ev.record(stream)
    sampler = ClockSampler(dev.index if dev.index is not None else 0) if sample_clocks else None
    barrier(world)
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.25)
    st.launches = 0
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        st.step(kev[i])
    stop.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    barrier(world)
    fa.fa_check_status(stream)
    launches = st.launches
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), world)
    fwd_ms = statistics.mean(e["f0"].elapsed_time(e["f1"]) for e in kev)
    bmain_ms = statistics.mean(e["b0"].elapsed_time(e["b1"]) for e in kev)
    return {"elapsed_ms": elapsed_ms, "fwd_ms": fwd_ms, "bwd_main_ms": bmain_ms, "clocks": clocks,
            "launches": launches}


def time_e2e(st: "StepSetup", steps: int, world: int):
    """The same step through the public API with host buffers: every step copies its inputs
    from pinned host memory and its results (O, LSE, dQ, dK, dV) back to pinned host memory.
    Device buffers are double-buffered and three streams (host->device, compute,
    device->host) overlap step k+1's upload and step k-1's download with step k's kernels;
    the timed region spans the first upload to the last download."""
    import torch
    dev, stream, host = st.dev, st.stream, st.host
    sets = []
    for _ in range(2):
        din = {n: torch.empty_like(t) for n, t in st.d.items()}
        dres = {"o": torch.empty_like(st.o), "lse": torch.empty_like(st.lse), "dq": torch.empty_like(st.dq),
                "dk": torch.empty_like(st.dk), "dv": torch.empty_like(st.dv)}
        sets.append((din, dres))
    host_out = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in sets[0][1].items()}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]

    def run(nsteps, t0=None, t1=None):
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
            st.forward(din["q"], din["k"], din["v"], dres["o"], dres["lse"])
            st.backward(din["q"], din["k"], din["v"], dres["o"], dres["lse"], din["dout"], dres["dq"], dres["dk"],
                        dres["dv"])
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

    run(2)
    torch.cuda.synchronize(dev)
    barrier(world)
    s2, t2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, s2, t2)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(s2.elapsed_time(t2), world)
    st.fa.fa_check_status(stream)
    return e2e_ms, h2d, d2h


def rates(w, t, world, steps):
    """TFLOP/s of the step, the forward and the fused main backward kernel."""
    from exact_attention_111_b200.inputs import attention_flops
    fwd_flops = attention_flops(w.B, w.H, w.N, w.d, w.causal, False)
    step_flops = attention_flops(w.B, w.H, w.N, w.d, w.causal, True)
    return {"step_flops": step_flops, "fwd_flops": fwd_flops, "bwd_flops": step_flops - fwd_flops,
            "value": aggregate_tflops(world, step_flops, steps, t["elapsed_ms"]),
            "fwd_tflops": fwd_flops / (t["fwd_ms"] * 1e-3) / 1e12,
            "bwd_main_tflops": (step_flops - fwd_flops) / (t["bwd_main_ms"] * 1e-3) / 1e12}


def run_ours(args, w, world, rank, local):
    import torch
    import exact_attention_111_b200 as fa

    fa.lib()  # fails loudly when the CUDA library is missing
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    st = StepSetup(args, w, rank, dev)
    t = time_device(st, args.steps, args.warmup, world, sample_clocks=True)
    r = rates(w, t, world, args.steps)
    e2e_steps = max(3, min(args.steps, 20))
    e2e_ms, h2d, d2h = time_e2e(st, e2e_steps, world)
    e2e_value = aggregate_tflops(world, r["step_flops"], e2e_steps, e2e_ms)
    main_splits = st.splits
    main_qsplits = st.qsplits
    del st
    torch.cuda.empty_cache()

    # The target point (d = 128, N = 16384, non-causal), same modes, device-timed like the main
    # line; every rank takes part so the barriers and max-over-ranks stay matched.
    target = None
    if args.target_point and w.name != TARGET_POINT:
        from exact_attention_111_b200.inputs import workloads
        wt = workloads()[TARGET_POINT]
        stt = StepSetup(args, wt, rank, dev)
        tt = time_device(stt, min(args.steps, 50), args.warmup, world, sample_clocks=True)
        rt = rates(wt, tt, world, min(args.steps, 50))
        target = (wt, tt, rt)
        del stt
        torch.cuda.empty_cache()

    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    peak_burst = float(peaks["bf16_tflops"])
    peak_sust = float(peaks.get("bf16_tflops_sustained", peak_burst))
    fwd_ms, bmain_ms = t["fwd_ms"], t["bwd_main_ms"]
    # dominant kernel: the one with the larger share of the step time
    if bmain_ms >= fwd_ms:
        dom, dom_tf, dom_flops = "bwd_main", r["bwd_main_tflops"], r["bwd_flops"]
    else:
        dom, dom_tf, dom_flops = "fwd", r["fwd_tflops"], r["fwd_flops"]
    traffic = stored_traffic(dom, w.name) if not (st_det(args) or args.dropout > 0) else None
    # The kernel is timed on its own by CUDA events around each launch: the burst peak applies.
    roofline = {"bound": "tensor", "achieved": dom_tf, "peak": peak_burst, "unit": "TFLOP/s",
                "frac": dom_tf / peak_burst, "traffic": traffic, "kernel": dom,
                "peak_source": f"bf16_tflops (burst) of {peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'profiling recipe fallback'})",
                "frac_of_sustained_peak": dom_tf / peak_sust,
                "frac_of_nominal_dense_bf16": dom_tf / NOMINAL_DENSE_BF16_TFLOPS,
                "algorithmic_flops_per_launch": dom_flops}
    value = r["value"]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t["elapsed_ms"] / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w, world),
                       **({"fwd_splits": main_splits, "fwd": "fa_fwd_splitkv (split forward + LSE merge, both inside "
                                                          "the fwd timing)"} if main_splits is not None else {}),
                       **({"bwd_query_splits": main_qsplits} if main_qsplits > 1 else {}),
                       **({"deterministic_bwd": "int64 fixed-point dQ accumulation"} if st_det(args) else {}),
                       **({"dropout_p": args.dropout,
                           "dropout": "fused, Philox4x32-10 mask regenerated in the backward"}
                          if args.dropout > 0 else {})),
        "fwd_tflops": r["fwd_tflops"], "fwd_ms": fwd_ms, "bwd_main_tflops": r["bwd_main_tflops"],
        "bwd_main_ms": bmain_ms,
        "fwd_bwd_frac_of_peak": value / world / peak_burst, "fwd_frac_of_peak": r["fwd_tflops"] / peak_burst,
        "fwd_bwd_frac_of_nominal": value / world / NOMINAL_DENSE_BF16_TFLOPS,
        "fwd_frac_of_nominal": r["fwd_tflops"] / NOMINAL_DENSE_BF16_TFLOPS,
        "peak_bf16_tflops_burst": peak_burst, "peak_source": peak_src,
        "nominal_dense_bf16_tflops": NOMINAL_DENSE_BF16_TFLOPS,
        "roofline": roofline,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps},
        "gpu_launches": t["launches"],
        "clocks": t["clocks"],
    }
    if target is not None:
        wt, tt, rt = target
        line["target_point"] = {
            "workload": wt.name, "steps": min(args.steps, 50), "ms_per_step": tt["elapsed_ms"] / min(args.steps, 50),
            "fwd_tflops": rt["fwd_tflops"], "fwd_bwd_tflops": rt["value"] / world,
            "bwd_main_tflops": rt["bwd_main_tflops"],
            "fwd_frac_of_peak": rt["fwd_tflops"] / peak_burst, "fwd_bwd_frac_of_peak": rt["value"] / world / peak_burst,
            "fwd_frac_of_nominal": rt["fwd_tflops"] / NOMINAL_DENSE_BF16_TFLOPS,
            "fwd_bwd_frac_of_nominal": rt["value"] / world / NOMINAL_DENSE_BF16_TFLOPS,
            "targets": "fwd >= 0.60 and fwd+bwd >= 0.45 of the dense BF16 peak",
            "gpu_launches": tt["launches"], "clocks": tt["clocks"]}
    if not args.no_cpu_baseline and world == 1:
        heads, el, flops = oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
                                "kind": "oracle",
                                "sample": f"{heads} whole (b, h) heads of {w.name}, forward + backward, "
                                          f"{el:.1f} s, fp64 numpy/BLAS"}
    print(json.dumps(line), flush=True)


def st_det(args) -> bool:
    return bool(args.deterministic)


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
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fwd-splits", type=int, default=None,
                    help="forward through fa_fwd_splitkv with this many key ranges (0: chosen for the "
                         "GPU; default: the workload's own setting)")
    ap.add_argument("--bwd-splits", type=int, default=None,
                    help="backward with each key tile's query range cut into this many ranges "
                         "(default: chosen for the GPU on the split-KV workloads, else none)")
    ap.add_argument("--dropout", type=float, default=0.0,
                    help="fused dropout probability in both passes (default 0: none)")
    ap.add_argument("--fp8", action="store_true",
                    help="time the FP8 (E4M3) forward alone on the workload (d = 128)")
    ap.add_argument("--deterministic", action="store_true",
                    help="backward in deterministic mode (bitwise repeatable dQ)")
    ap.add_argument("--no-target-point", dest="target_point", action="store_false",
                    help=f"skip the extra timing of {TARGET_POINT} reported as target_point")
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
