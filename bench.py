#!/usr/bin/env python
"""Benchmark of the tensor-parallel two-projection MLP on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config decode_bs1|decode_bs32|prefill|sweep|tiny] [--tokens T] [--tp P]
                    [--plan auto|gemv|simt|tc]

One step = one forward of the whole hot path (first projection + activation,
second projection with the ranks' partial sums reduced on the device) over one
batch of seeded synthetic input, on weights packed once before timing.  The
default workload is decode at batch 1 (bf16 SwiGLU, d_model 8192, d_ff 28672,
8 ranks' shards on one GPU).  The weights (1.41 GB) are far larger than L2, so
every step re-reads them from HBM; no L2 flush is needed.

Rank 0 prints one JSON line.  With N > 1 (torchrun) each GPU runs an
independent replica on its own batch (data-parallel replicas: no collective on
the data path); the reported time is the max over ranks.

--impl reference times the oracle (plain fp64 C loops on the host cores) on a
bounded sample of the same workload; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sharded-MLP tokens/s; decode HBM GB/s & prefill TFLOP/s vs B200 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="decode_bs1")
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--tp", type=int, default=None)
    ap.add_argument("--plan", default="auto")
    ap.add_argument("--splitk", choices=["auto", "in_kernel", "separate"], default="auto",
                    help="how the skinny tensor-core tiling finishes split tiles")
    ap.add_argument("--d-model", type=int, default=None, help="override (small cases for profiling)")
    ap.add_argument("--d-ff", type=int, default=None, help="override (small cases for profiling)")
    ap.add_argument("--api", choices=["packed", "shard"], default="packed",
                    help="packed: weights packed once, tp_mlp_forward_packed; shard: tp_mlp_forward on the shards")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay percentiles")
    return ap.parse_args()


def resolve(args):
    from tensor_sharded_mlp_b200 import inputs
    c = dict(inputs.CONFIGS[args.config])
    T = c["tokens"]
    if isinstance(T, tuple):
        T = args.tokens if args.tokens is not None else T[-1]
    elif args.tokens is not None:
        T = args.tokens
    tp = c["tp"]
    if isinstance(tp, tuple):
        tp = args.tp if args.tp is not None else tp[-1]
    elif args.tp is not None:
        tp = args.tp
    c.update(tokens=T, tp=tp)
    small = ""
    if args.d_model is not None or args.d_ff is not None:
        c["d_model"] = args.d_model or c["d_model"]
        c["d_ff"] = args.d_ff or c["d_ff"]
        small = " [reduced size for profiling]"
    c["workload"] = (f"{args.config}{small}: {c['dtype']} {c['act']} MLP, tokens={T}, d_model={c['d_model']}, "
                     f"d_ff={c['d_ff']}, tp={tp} shards on one GPU, X~N(0,1), "
                     f"weights~N(0,{'1/fan_in' if c['init'] == 'fan_in' else str(c['init']) + '^2'}), "
                     f"seed {c['seed']}")
    return c


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernel source."""
    from tensor_sharded_mlp_b200.counts import kernel_source_hash
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    e = rec.get(f"{kernel}|{workload}")
    if not e or e.get("source_hash") != kernel_source_hash(kernel.split(":")[0]):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples = []
        self.period = period_s
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report no clocks rather than invent them
            self.err = str(e)
        self.window = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), sm, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": getattr(self, "err", "no samples")}
        sel = self.samples
        if self.window:
            w = [s for s in self.samples if self.window[0] <= s[0] <= self.window[1]]
            if len(w) >= 3:
                sel = w
        mask = 0
        for s in sel:
            mask |= s[2]
        reasons = [n for b, n in self.REASONS.items() if mask & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[1] for s in sel), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sel),
                "window": "timed region" if sel is not self.samples else "warm-up + timed region"}


def _oracle_rate(p, A, Bs, act, budget_s, max_calls):
    import oracle
    calls, t_total = 0, 0.0
    while calls < max_calls and t_total < budget_s:
        t0 = time.perf_counter()
        oracle.tp_mlp_sharded(p.x, A, Bs, act)
        t_total += time.perf_counter() - t0
        calls += 1
    return p.tokens * calls / t_total, calls, t_total


def oracle_baseline(p, A, Bs, act, budget_s=12.0, max_calls=50):
    """Time the oracle as it stands on a bounded sample: whole calls until the budget is spent.
    With more than one token the oracle's OpenMP loop can use several cores, so it is
    also timed on one core; with one token both are the same run."""
    import oracle
    T = p.tokens
    nproc = os.cpu_count()
    try:
        affinity = len(os.sched_getaffinity(0))
    except AttributeError:
        affinity = nproc
    threads = min(oracle.max_threads(), T)
    value, calls, t_total = _oracle_rate(p, A, Bs, act, budget_s, max_calls)
    out = {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
           "host_nproc": nproc, "host_affinity": affinity,
           "sample": f"{calls} full forward(s) of this workload ({T} token(s) each) on the host, "
                     f"{t_total:.1f} s; the oracle runs OpenMP over tokens"}
    if threads > 1:
        oracle.set_threads(1)
        try:
            v1, c1, t1 = _oracle_rate(p, A, Bs, act, budget_s / 2, max_calls)
        finally:
            oracle.set_threads(oracle.max_threads())
        out["one_core"] = {"value": v1, "sample": f"{c1} full forward(s), {t1:.1f} s"}
    return out


def graph_replay_stats(fwd, K, W):
    """Per-step device time of the forward captured once in a CUDA graph and
    replayed K times, each replay bracketed by its own events (so a replay does
    not overlap the previous one): median and 10th / 90th percentiles, in us."""
    import torch
    gs = torch.cuda.Stream()
    gs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(gs):
        fwd()
    gs.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=gs):
        fwd()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    with torch.cuda.stream(gs):
        for _ in range(W):
            g.replay()
        for a, b in ev:
            a.record(gs)
            g.replay()
            b.record(gs)
    gs.synchronize()
    d = sorted(a.elapsed_time(b) * 1e3 for a, b in ev)
    del g

    def pct(q):
        return d[min(len(d) - 1, int(round(q * (len(d) - 1))))]
    return {"p10_us": pct(0.1), "p50_us": pct(0.5), "p90_us": pct(0.9), "replays": K,
            "timer": "CUDA events around each replay of the captured forward"}


def run_fused_norm_reference(args):
    """Reference arm of the fused step: the oracle on whole rows, bounded."""
    if int(os.environ.get("RANK", 0)) != 0:
        return 0
    from tensor_sharded_mlp_b200 import inputs
    c = _fused_norm_config(args)
    fi = inputs.generate_fused_norm(c["tokens"], c["d_model"], c["tp"], c["dtype"], c["seed"], c["eps"])
    budget = 150.0 / max(1, args.steps + args.warmup)
    rates = []
    for i in range(args.warmup + args.steps):
        v, rows, tt = fused_norm_oracle_rate(fi, budget)
        if i >= args.warmup:
            rates.append((rows, tt))
    rows = sum(r for r, _ in rates)
    tt = sum(t for _, t in rates)
    value = rows / tt
    sample = f"each step: the oracle on whole token rows for about {budget:.1f} s ({rows} rows in all)"
    line = {"impl": "reference", "metric": FUSED_NORM_METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": c["workload"], "tokens": c["tokens"], "d_model": c["d_model"], "tp": c["tp"],
                       "parallelism": "host oracle"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_reference(args):
    rank = int(os.environ.get("RANK", 0))
    if rank != 0:
        return 0
    import oracle
    from tensor_sharded_mlp_b200 import inputs
    c = resolve(args)
    p = inputs.generate(c["tokens"], c["d_model"], c["d_ff"], c["act"], c["dtype"], c["seed"], c["init"])
    A, Bs = p.shards(c["tp"])
    T, P = c["tokens"], c["tp"]
    # sample: the first t_s tokens and the first r_s of the P ranks (work is linear in both)
    t_s = min(T, 64)
    oracle.tp_mlp_sharded(p.x[:t_s], A[:1], Bs[:1], c["act"])          # warm the code path
    t0 = time.perf_counter()
    oracle.tp_mlp_sharded(p.x[:t_s], A[:1], Bs[:1], c["act"])
    per_rank = time.perf_counter() - t0
    budget = 150.0 / max(1, args.steps + args.warmup)
    r_s = max(1, min(P, int(budget / max(per_rank, 1e-6))))
    for _ in range(args.warmup):
        oracle.tp_mlp_sharded(p.x[:t_s], A[:r_s], Bs[:r_s], c["act"])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.tp_mlp_sharded(p.x[:t_s], A[:r_s], Bs[:r_s], c["act"])
    dt = time.perf_counter() - t0
    work_tokens = t_s * r_s / P * args.steps
    value = work_tokens / dt
    cores = min(oracle.max_threads(), t_s)
    sample = (f"each step: the oracle on the first {t_s} of {T} token(s) and {r_s} of {P} ranks' shards "
              f"({r_s}/{P} of the weights); tokens/s counts {t_s}*{r_s}/{P} tokens per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": c["workload"], "tokens": T, "d_model": c["d_model"],
                                             "d_ff": c["d_ff"], "tp": P, "act": c["act"],
                                             "parallelism": "host oracle"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


FUSED_NORM_METRIC = "fused TP all-reduce + residual add + RMSNorm: token rows/s; HBM GB/s vs B200 peak"


def _fused_norm_config(args):
    from tensor_sharded_mlp_b200 import inputs
    c = dict(inputs.FUSED_NORM_CONFIGS[args.config])
    if args.tokens is not None:
        c["tokens"] = args.tokens
    if args.tp is not None:
        c["tp"] = args.tp
    c["workload"] = (f"{args.config}: all-reduce of {c['tp']} fp32 rank partials + residual add + RMSNorm "
                     f"({c['dtype']} residual/gamma/outputs), tokens={c['tokens']}, d_model={c['d_model']}, "
                     f"eps={c['eps']}, partials and residual ~N(0,1), gamma ~1+0.1 N(0,1), seed {c['seed']}")
    return c


def fused_norm_oracle_rate(fi, budget_s):
    """The oracle as it stands on whole token rows, for about budget_s seconds."""
    import oracle
    T = fi.residual.shape[0]
    rows, t_total, n = 0, 0.0, 1
    while t_total < budget_s:
        n = min(T, n)
        t0 = time.perf_counter()
        oracle.allreduce_residual_rmsnorm(fi.partials[:, :n], fi.residual[:n], fi.gamma, fi.eps)
        t_total += time.perf_counter() - t0
        rows += n
        n *= 2
    return rows / t_total, rows, t_total


def run_fused_norm(args):
    """The fused all-reduce + residual + RMSNorm step ("7.4 推理侧并行" §7.4.2):
    one tp_mlp_allreduce_residual_rmsnorm launch per step."""
    import numpy as np
    import torch

    from tensor_sharded_mlp_b200 import binding, counts, inputs, replicas

    rank, world, local = replicas.rank_env()
    torch.cuda.set_device(local)
    replicas.init("nccl", torch.device("cuda", local))
    c = _fused_norm_config(args)
    T, d, P, dt, eps = c["tokens"], c["d_model"], c["tp"], c["dtype"], c["eps"]
    fi = inputs.generate_fused_norm(T, d, P, dt, c["seed"], eps)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    step_bytes = counts.fused_norm_bytes(P, T, d, dt)
    # inputs smaller than L2 are rotated through enough copies to exceed it
    copies = max(1, -(-2 * 126 * 2 ** 20 // step_bytes))
    p0 = torch.from_numpy(fi.partials).cuda()
    r0 = torch.from_numpy(fi.residual).cuda().to(tdt)
    g = torch.from_numpy(fi.gamma).cuda().to(tdt)
    sets = [(p0, r0)] + [(p0.clone(), r0.clone()) for _ in range(copies - 1)]
    y = torch.empty(T, d, dtype=tdt, device="cuda")
    ro = torch.empty(T, d, dtype=tdt, device="cuda")
    K, W = args.steps, max(3, args.warmup)

    def step(i):
        pi, ri = sets[i % copies]
        binding.tp_mlp_allreduce_residual_rmsnorm(pi, ri, g, eps, y, ro)

    for i in range(W):
        step(i)
    torch.cuda.synchronize()
    # A launch from Python costs more host time than a decode-sized kernel takes
    # on the GPU, so the K steps are captured once in a CUDA graph (the pages'
    # remedy for launch overhead, "7.4 推理侧并行" §7.4.2) and the timed region
    # is one replay of it; the host-bound per-call time is reported beside it.
    gs = torch.cuda.Stream()
    gs.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=gs):
        for i in range(K):
            step(i)
    for _ in range(W):
        graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.1)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    replicas.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    start.record(stream)
    graph.replay()
    end.record(stream)
    replicas.barrier()
    torch.cuda.synchronize()
    sampler.mark(t0, time.perf_counter())
    elapsed_ms = replicas.max_over_ranks(start.elapsed_time(end))
    launch_ms = start.elapsed_time(end) / K    # back-to-back launches inside the graph
    # the same K launches issued from Python one by one (host-bound when small)
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(stream)
    for i in range(K):
        step(i)
    h1.record(stream)
    torch.cuda.synchronize()
    api_ms = h0.elapsed_time(h1) / K
    del graph
    # the same step unfused, with library ops: sum over ranks, residual add, RMSNorm
    def unfused(i):
        pi, ri = sets[i % copies]
        h = (pi.sum(dim=0) + ri.float()).to(tdt)
        return torch.nn.functional.rms_norm(h.float(), (d,), weight=g.float(), eps=eps).to(tdt), h
    for i in range(W):
        unfused(i)
    ue = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i, (a, b) in enumerate(ue):
        a.record(stream)
        unfused(i)
        b.record(stream)
    torch.cuda.synchronize()
    unfused_ms = statistics.fmean(a.elapsed_time(b) for a, b in ue)
    # end to end: pinned host inputs in, both outputs back, every step
    e2e = None
    if not args.no_e2e:
        hp = torch.from_numpy(fi.partials).pin_memory()
        hr = r0.cpu().pin_memory()
        hy = torch.empty(T, d, dtype=tdt).pin_memory()
        hro = torch.empty(T, d, dtype=tdt).pin_memory()
        dp, dr = sets[0]
        for _ in range(W):
            dp.copy_(hp, non_blocking=True)
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        for _ in range(K):
            dp.copy_(hp, non_blocking=True)
            dr.copy_(hr, non_blocking=True)
            binding.tp_mlp_allreduce_residual_rmsnorm(dp, dr, g, eps, y, ro)
            hy.copy_(y, non_blocking=True)
            hro.copy_(ro, non_blocking=True)
            stream.synchronize()
        e2.record(stream)
        e2.synchronize()
        e2e_ms = replicas.max_over_ranks(s2.elapsed_time(e2))
        e2e = {"value": replicas.whole_job_rate(T, K, world, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": hp.numel() * 4 + hr.numel() * hr.element_size(),
               "d2h_bytes_per_step": 2 * hy.numel() * hy.element_size(),
               "api": "binding.tp_mlp_allreduce_residual_rmsnorm with pinned host buffers, synchronize per step"}
    sampler.stop()
    peaks, src = load_peaks()
    achieved = step_bytes / (launch_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": recorded_traffic("fused_norm:norm", args.config),
                "kernel": "allreduce_norm_kernel", "kernel_ms": launch_ms, "algorithmic_per_launch": step_bytes,
                "peak_source": f"hbm_gbs ({src})"}
    ms = elapsed_ms / K
    line = {"metric": FUSED_NORM_METRIC, "value": replicas.whole_job_rate(T, K, world, elapsed_ms),
            "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dt, "data": "synthetic",
            "config": {"workload": c["workload"], "tokens": T, "d_model": d, "tp": P, "eps": eps,
                       "parallelism": "replicas" if world > 1 else "single GPU",
                       "l2": (f"{copies} input copies rotated ({copies * step_bytes / 2 ** 20:.0f} MiB > L2)"
                              if copies > 1 else "inputs larger than L2")},
            "step_hbm_gbs": step_bytes / (ms / 1e3) / 1e9, "roofline": roofline, "gpu_launches": K,
            "clocks": sampler.summary(), "e2e": e2e,
            "timer": "CUDA events around one replay of a CUDA graph holding the K launches",
            "python_call_us": api_ms * 1e3,
            "unfused_library_ops": {"ms": unfused_ms, "ops": "torch sum over ranks, add, rms_norm",
                                    "algorithmic_bytes": counts.unfused_norm_bytes(P, T, d, dt)}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, rows, tt = fused_norm_oracle_rate(fi, 10.0)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"{rows} token rows of this workload on one host core, {tt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    replicas.finish()
    return 0


def main():
    args = parse()
    from tensor_sharded_mlp_b200 import inputs as _inputs
    if args.config in _inputs.FUSED_NORM_CONFIGS:
        if args.impl == "reference":
            return run_fused_norm_reference(args)
        return run_fused_norm(args)
    if args.impl == "reference":
        return run_reference(args)

    import numpy as np
    import torch

    from tensor_sharded_mlp_b200 import binding, counts, inputs, replicas

    rank, world, local = replicas.rank_env()
    torch.cuda.set_device(local)
    replicas.init("nccl", torch.device("cuda", local))
    c = resolve(args)
    T, d, f, tp, act, dt = c["tokens"], c["d_model"], c["d_ff"], c["tp"], c["act"], c["dtype"]
    p = inputs.generate(T, d, f, act, dt, c["seed"], c["init"])
    A, Bs = p.shards(tp)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32

    def up(a):
        return torch.from_numpy(a).cuda().to(tdt).contiguous()

    m = binding.TpMlp(d, f, tp, act, dt, max_tokens=T)
    m.set_plan(args.plan)
    m.set_splitk(args.splitk)
    Ad, Bd = [up(a) for a in A], [up(b) for b in Bs]
    packed = m.pack(Ad, Bd)
    if args.api == "packed":
        del Ad, Bd
        fwd = lambda: m.forward_packed(x, packed, out=out)            # noqa: E731
    else:
        fwd = lambda: m.forward(x, Ad, Bd, out=out)                   # noqa: E731
    x = up(p.x)
    out = torch.empty(T, d, dtype=tdt, device="cuda")
    torch.cuda.synchronize()

    def barrier():
        replicas.barrier()
        torch.cuda.synchronize()

    K, W = args.steps, max(3, args.warmup)
    for _ in range(W):
        fwd()
    nk = m.last_launches
    plan = m.last_plan
    # the library marks phases: before the first projection's kernels, between
    # the projections and after the second's (a phase may be more than one kernel)
    nph = 2
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nph + 1)] for _ in range(K)]
    stream = torch.cuda.current_stream()
    for row in ev:
        for e in row:
            e.record(stream)
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.1)
    # Timed region: K clean steps (kernels back to back, so each may overlap the
    # previous one's tail through programmatic dependent launch).
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    t0 = time.perf_counter()
    start.record(stream)
    for i in range(K):
        fwd()
    end.record(stream)
    barrier()
    t1 = time.perf_counter()
    sampler.mark(t0, t1)
    elapsed_ms = start.elapsed_time(end)
    # Per-kernel durations: the same K steps again with the library recording
    # events on the launch stream before, between and after its kernels.
    for i in range(K):
        binding.tp_mlp_set_profile_events(m.h, ev[i])
        fwd()
    binding.tp_mlp_set_profile_events(m.h, None)
    barrier()
    kern_ms = [statistics.fmean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K)) for j in range(nph)]
    elapsed_ms = replicas.max_over_ranks(elapsed_ms)
    graph_steps = None
    if not args.no_graph:
        graph_steps = graph_replay_stats(fwd, max(K, 50), W)
        barrier()

    # end to end through the public API with host buffers (pinned), copies inside
    # the region: binding.GraphStep replays H2D(x) + forward + D2H(out) as one
    # CUDA graph and waits for the result every step, as a decode loop must.
    e2e = None
    if not args.no_e2e and args.api == "packed":
        step = binding.GraphStep(m, packed, T)
        step.x_host.copy_(x.cpu())
        for _ in range(W):
            step()
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(step.stream)
        for _ in range(K):
            step()                    # replay + wait for the result on the host
        e2.record(step.stream)
        e2.synchronize()
        e2e_ms = replicas.max_over_ranks(s2.elapsed_time(e2))
        ref_out = out.cpu()
        e2e_ok = bool(torch.equal(step.out_host, ref_out))
        e2e = {"value": replicas.whole_job_rate(T, K, world, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": step.x_host.numel() * step.x_host.element_size(),
               "d2h_bytes_per_step": step.out_host.numel() * step.out_host.element_size(),
               "api": "binding.GraphStep (CUDA graph: H2D x, tp_mlp_forward_packed, D2H out, synchronize)",
               "timer": "CUDA events on the step's stream around K steps, host waits included",
               "matches_device_result": e2e_ok}
        del step
    sampler.stop()

    value = replicas.whole_job_rate(T, K, world, elapsed_ms)
    peaks, src = load_peaks()
    # roofline of the dominant kernel (largest share of the step)
    j = int(np.argmax(kern_ms))
    names = ["first projection + activation", "second projection + rank sum"]
    if plan in ("tc_wide", "tc_wide256"):
        bound, unit = "tensor", "TFLOP/s"
        work = counts.gemm1_flops(T, d, f, act) if j == 0 else counts.gemm2_flops(T, f, d)
        achieved = work / (kern_ms[j] / 1e3) / 1e12
        peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
        peak_note = f"bf16_tflops_sustained ({src})"
    else:
        bound, unit = "hbm", "GB/s"
        work = counts.gemm1_bytes(T, d, f, act, dt) if j == 0 else counts.gemm2_bytes(T, f, d, dt)
        achieved = work / (kern_ms[j] / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        peak_note = f"hbm_gbs ({src})"
    kname = f"{plan}:{'first' if j == 0 else 'second'}"
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                "traffic": recorded_traffic(kname, args.config), "kernel": names[j] + (" (GEMM + split-tile reduction kernel)" if nk > 2 and plan == "tc_skinny" else ""),
                "kernel_ms": kern_ms[j], "algorithmic_per_launch": work, "peak_source": peak_note,
                "kernel_ms_all": kern_ms}
    step_bytes = counts.algorithmic_bytes(T, d, f, d, act, dt)
    step_flops = counts.forward_flops(T, d, f, d, act)
    ms = elapsed_ms / K
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": dt, "data": "synthetic",
            "config": {"workload": c["workload"], "tokens": T, "d_model": d, "d_ff": f, "tp": tp, "act": act,
                       "plan": plan, "splitk": args.splitk, "api": args.api, "parallelism": "replicas" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2: every step re-reads %.2f GB of weights" % (step_bytes / 1e9)},
            "step_hbm_gbs": step_bytes / (ms / 1e3) / 1e9, "step_tflops": step_flops / (ms / 1e3) / 1e12,
            "roofline": roofline, "gpu_launches": K * nk, "clocks": sampler.summary(), "e2e": e2e,
            "graph_step": graph_steps}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_baseline(p, A, Bs, act)
    if rank == 0:
        print(json.dumps(line), flush=True)
    replicas.finish()
    return 0


if __name__ == "__main__":
    sys.exit(main())
