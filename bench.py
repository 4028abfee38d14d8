#!/usr/bin/env python
"""Benchmark of the tensor-parallel two-projection MLP on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config decode_bs1|decode_bs32|prefill|sweep|tiny] [--tokens T] [--tp P]
                    [--plan auto|simt|gemv|tc|tc_skinny|tc_fused|tc_wide|tc_wide256|tc_pair|tc_pair2] [--api packed|shard]
                    [--splitk auto|in_kernel|separate|cluster] [--no-e2e] [--no-cpu-baseline] [--no-graph]
                    [--configs auto|all|none]
    python bench.py --config fused_norm_decode_bs32|fused_norm_prefill|
                             attn_merge_decode_bs32|attn_merge_decode_bs256 [...]
    torchrun --nproc-per-node N bench.py --config xgpu_decode_bs32 [...]

One step = one forward of the whole hot path (first projection + activation,
second projection with the ranks' partial sums reduced on the device) over one
batch of seeded synthetic input, on weights packed once before timing.  The
default workload is decode at batch 1 (bf16 SwiGLU, d_model 8192, d_ff 28672,
8 ranks' shards on one GPU).  The weights (1.41 GB) are far larger than L2, so
every step re-reads them from HBM; no L2 flush is needed.

The default invocation also times the rest of the metric in the same run and
adds it to the line as "configs": decode at batch 32, prefill (8192 tokens,
tp 8; TFLOP/s against the bf16 peak) and the TP x token sweep at 16, 128 and
1024 tokens (tp 8), each with its own inputs, steps, per-kernel roofline,
clock record and CPU baseline (--configs none skips them).

Rank 0 prints one JSON line.  With N > 1 (torchrun) each GPU runs an
independent replica on its own batch (data-parallel replicas: no collective on
the data path); the reported time is the max over ranks.

--impl reference times the oracle (plain fp64 C loops on the host cores) on a
bounded sample of the same workload; under torchrun only rank 0 runs it.

The fused_norm_* and attn_merge_* configs time the two other operators (the
all-reduce fused with residual add and RMSNorm; the merge of attention
partials across KV shards): one launch per step, the K steps captured in a
CUDA graph, inputs smaller than L2 rotated through enough copies to exceed it.

The xgpu_decode_bs32 config runs tensor parallelism across GPUs (one rank per
GPU under torchrun, tp = the number of ranks) and times the fused one-shot
all-reduce step against each rank's partial followed by NCCL's all_reduce.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

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
    ap.add_argument("--config", default="decode_bs1",
                    help="MLP: tiny, decode_bs1, decode_bs32, sweep, prefill; other operators: "
                         "fused_norm_decode_bs32, fused_norm_prefill, attn_merge_decode_bs32, "
                         "attn_merge_decode_bs256; across GPUs (torchrun): xgpu_decode_bs32")
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--tp", type=int, default=None)
    ap.add_argument("--plan", default="auto")
    ap.add_argument("--splitk", choices=["auto", "in_kernel", "separate", "cluster"], default="auto",
                    help="how the skinny tensor-core tiling finishes split tiles")
    ap.add_argument("--d-model", type=int, default=None, help="override (small cases for profiling)")
    ap.add_argument("--d-ff", type=int, default=None, help="override (small cases for profiling)")
    ap.add_argument("--api", choices=["packed", "shard"], default="packed",
                    help="packed: weights packed once, tp_mlp_forward_packed; shard: tp_mlp_forward on the shards")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip timing the oracle on the host")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay percentiles")
    ap.add_argument("--configs", choices=["auto", "all", "none"], default="auto",
                    help="also time decode_bs32, prefill (tp 8) and the sweep at T=16/128/1024 (tp 8) in the same "
                         "run, each in the 'configs' block of the JSON line; auto: only for the default "
                         "invocation (decode_bs1, nothing overridden), on one GPU")
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


def _oracle_rate(x, A, Bs, act, budget_s, max_calls):
    import oracle
    calls, t_total = 0, 0.0
    while calls < max_calls and t_total < budget_s:
        t0 = time.perf_counter()
        oracle.tp_mlp_sharded(x, A, Bs, act)
        t_total += time.perf_counter() - t0
        calls += 1
    return x.shape[0] * calls / t_total, calls, t_total


def oracle_baseline(p, A, Bs, act, budget_s=12.0, max_calls=50, sample_rows=None, one_core=True):
    """Time the oracle as it stands on a bounded sample: whole calls until the budget is spent
    (at least one).  With sample_rows, each call takes that many seeded-sampled token rows
    instead of the whole batch.  With more than one token the oracle's OpenMP loop can use
    several cores, so it is also timed on one core; with one token both are the same run."""
    import oracle
    T = p.tokens
    nproc = os.cpu_count()
    try:
        affinity = len(os.sched_getaffinity(0))
    except AttributeError:
        affinity = nproc
    x = p.x
    what = f"full forward(s) of this workload ({T} token(s) each)"
    if sample_rows is not None and sample_rows < T:
        rows = p.sample_rows(sample_rows)
        x = np.ascontiguousarray(p.x[rows])
        what = f"forward(s) of {len(rows)} seeded-sampled of the {T} token rows"
    n = x.shape[0]
    threads = min(oracle.max_threads(), n)
    value, calls, t_total = _oracle_rate(x, A, Bs, act, budget_s, max_calls)
    out = {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
           "host_nproc": nproc, "host_affinity": affinity,
           "sample": f"{calls} {what} on the host, {t_total:.1f} s; the oracle runs OpenMP over tokens"}
    if threads > 1 and one_core:
        oracle.set_threads(1)
        try:
            x1 = x[:max(1, n // threads)]
            v1, c1, t1 = _oracle_rate(x1, A, Bs, act, budget_s / 2, max_calls)
        finally:
            oracle.set_threads(oracle.max_threads())
        out["one_core"] = {"value": v1, "sample": f"{c1} forward(s) of {x1.shape[0]} of those rows, {t1:.1f} s"}
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
ATTN_MERGE_METRIC = "DCP merge of KV-shard attention partials: query rows/s; HBM GB/s vs B200 peak"


class FusedNormOp:
    """The all-reduce + residual add + RMSNorm step ("7.4 推理侧并行" §7.4.2)."""
    metric = FUSED_NORM_METRIC
    kernel = "allreduce_norm_kernel"
    family = "fused_norm"
    library_ops = "torch sum over ranks, add, rms_norm"

    def __init__(self, args):
        from tensor_sharded_mlp_b200 import inputs
        c = dict(inputs.FUSED_NORM_CONFIGS[args.config])
        if args.tokens is not None:
            c["tokens"] = args.tokens
        if args.tp is not None:
            c["tp"] = args.tp
        self.c = c
        self.units = c["tokens"]
        self.dtype = c["dtype"]
        self.workload = (f"{args.config}: all-reduce of {c['tp']} fp32 rank partials + residual add + RMSNorm "
                         f"({c['dtype']} residual/gamma/outputs), tokens={c['tokens']}, d_model={c['d_model']}, "
                         f"eps={c['eps']}, partials and residual ~N(0,1), gamma ~1+0.1 N(0,1), seed {c['seed']}")
        self.config = {"tokens": c["tokens"], "d_model": c["d_model"], "tp": c["tp"], "eps": c["eps"]}
        self.host = inputs.generate_fused_norm(c["tokens"], c["d_model"], c["tp"], c["dtype"], c["seed"], c["eps"])

    def step_bytes(self):
        from tensor_sharded_mlp_b200 import counts
        return counts.fused_norm_bytes(self.c["tp"], self.c["tokens"], self.c["d_model"], self.dtype)

    def library_bytes(self):
        from tensor_sharded_mlp_b200 import counts
        return counts.unfused_norm_bytes(self.c["tp"], self.c["tokens"], self.c["d_model"], self.dtype)

    def device(self, torch, tdt):
        """(inputs that differ per rotated copy, fixed inputs, outputs)."""
        p = torch.from_numpy(self.host.partials).cuda()
        r = torch.from_numpy(self.host.residual).cuda().to(tdt)
        g = torch.from_numpy(self.host.gamma).cuda().to(tdt)
        T, d = self.c["tokens"], self.c["d_model"]
        return (p, r), (g,), (torch.empty(T, d, dtype=tdt, device="cuda"), torch.empty(T, d, dtype=tdt, device="cuda"))

    def launch(self, binding, ins, fixed, outs):
        binding.tp_mlp_allreduce_residual_rmsnorm(ins[0], ins[1], fixed[0], self.c["eps"], outs[0], outs[1])

    def library(self, torch, ins, fixed):
        p, r = ins
        h = (p.sum(dim=0) + r.float()).to(r.dtype)
        return torch.nn.functional.rms_norm(h.float(), (h.shape[1],), weight=fixed[0].float(),
                                            eps=self.c["eps"]).to(r.dtype), h

    def oracle_rate(self, budget_s):
        import oracle
        fi, T = self.host, self.c["tokens"]
        rows, t_total, n = 0, 0.0, 1
        while t_total < budget_s:
            n = min(T, n)
            t0 = time.perf_counter()
            oracle.allreduce_residual_rmsnorm(fi.partials[:, :n], fi.residual[:n], fi.gamma, fi.eps)
            t_total += time.perf_counter() - t0
            rows += n
            n *= 2
        return rows / t_total, rows, t_total


class AttnMergeOp:
    """The merge of KV shards' partial attention results ("LLM 推理并行化" §三 4), DCP)."""
    metric = ATTN_MERGE_METRIC
    kernel = "attn_merge_kernel"
    family = "attn_merge"
    library_ops = "torch max, exp, weighted sums and division over ranks"

    def __init__(self, args):
        from tensor_sharded_mlp_b200 import inputs
        c = dict(inputs.ATTN_MERGE_CONFIGS[args.config])
        if args.tokens is not None:
            c["tokens"] = args.tokens
        if args.tp is not None:
            c["tp"] = args.tp
        self.c = c
        self.rows = c["tokens"] * c["heads"]
        self.units = self.rows
        self.dtype = c["dtype"]
        self.workload = (f"{args.config}: merge of {c['tp']} KV shards' attention partials, {c['tokens']} decode "
                         f"queries x {c['heads']} heads of {c['head_dim']} ({c['dtype']} weighted sums, fp32 maxima "
                         f"and sums), maxima ~N(0,4), sums ~1+U*(keys_per_rank-1) with {c['keys_per_rank']} keys "
                         f"per rank, weighted ~N(0,1)*sqrt(sum), seed {c['seed']}")
        self.config = {"tokens": c["tokens"], "heads": c["heads"], "head_dim": c["head_dim"], "tp": c["tp"]}
        self.host = inputs.generate_attn_merge(c["tp"], self.rows, c["head_dim"], c["dtype"], c["seed"],
                                               c["keys_per_rank"])

    def step_bytes(self):
        e = 4 if self.dtype == "f32" else 2
        P, D = self.c["tp"], self.c["head_dim"]
        return P * self.rows * (8 + D * e) + self.rows * D * e

    def library_bytes(self):
        return None

    def device(self, torch, tdt):
        m = torch.from_numpy(self.host.maximum).cuda()
        s = torch.from_numpy(self.host.exp_sum).cuda()
        w = torch.from_numpy(self.host.weighted).cuda().to(tdt)
        return (m, s, w), (), (torch.empty(self.rows, self.c["head_dim"], dtype=tdt, device="cuda"),)

    def launch(self, binding, ins, fixed, outs):
        binding.tp_mlp_merge_attention_partials(ins[0], ins[1], ins[2], outs[0])

    def library(self, torch, ins, fixed):
        m, s, w = ins
        c = torch.exp(m - m.max(dim=0, keepdim=True).values)
        return ((c[:, :, None] * w.float()).sum(dim=0) / (c * s).sum(dim=0)[:, None]).to(w.dtype)

    def oracle_rate(self, budget_s):
        import oracle
        a = self.host
        rows, t_total, n = 0, 0.0, 64
        while t_total < budget_s:
            n = min(self.rows, n)
            t0 = time.perf_counter()
            oracle.merge_attention_partials(a.maximum[:, :n], a.exp_sum[:, :n], a.weighted[:, :n])
            t_total += time.perf_counter() - t0
            rows += n
            n *= 2
        return rows / t_total, rows, t_total


def small_op(args):
    from tensor_sharded_mlp_b200 import inputs
    if args.config in inputs.FUSED_NORM_CONFIGS:
        return FusedNormOp(args)
    if args.config in inputs.ATTN_MERGE_CONFIGS:
        return AttnMergeOp(args)
    return None


def run_small_op(args, op):
    """One launch of a small memory-bound operator per step."""
    import torch

    from tensor_sharded_mlp_b200 import binding, replicas

    rank, world, local = replicas.rank_env()
    torch.cuda.set_device(local)
    replicas.init("nccl", torch.device("cuda", local))
    tdt = torch.bfloat16 if op.dtype == "bf16" else torch.float32
    step_bytes = op.step_bytes()
    # inputs smaller than L2 are rotated through enough copies to exceed it
    copies = max(1, -(-2 * 126 * 2 ** 20 // step_bytes))
    ins0, fixed, outs = op.device(torch, tdt)
    sets = [ins0] + [tuple(t.clone() for t in ins0) for _ in range(copies - 1)]
    K, W = args.steps, max(3, args.warmup)

    def step(i):
        op.launch(binding, sets[i % copies], fixed, outs)

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
    del graph
    # the same K launches issued from Python one by one (host-bound when small)
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(stream)
    for i in range(K):
        step(i)
    h1.record(stream)
    torch.cuda.synchronize()
    api_ms = h0.elapsed_time(h1) / K
    # the same step with library ops (several kernels), for comparison
    for i in range(W):
        op.library(torch, sets[i % copies], fixed)
    u0, u1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    u0.record(stream)
    for i in range(K):
        op.library(torch, sets[i % copies], fixed)
    u1.record(stream)
    torch.cuda.synchronize()
    library_ms = u0.elapsed_time(u1) / K
    # end to end: pinned host inputs in, outputs back, every step
    e2e = None
    if not args.no_e2e:
        host_in = [t.cpu().pin_memory() for t in sets[0]]
        host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for it in range(W + K):
            if it == W:
                s2.record(stream)
            for dst, src in zip(sets[0], host_in):
                binding.tp_mlp_copy_async(dst, src)
            op.launch(binding, sets[0], fixed, outs)
            for dst, src in zip(host_out, outs):
                binding.tp_mlp_copy_async(dst, src)
            stream.synchronize()
        e2.record(stream)
        e2.synchronize()
        e2e_ms = replicas.max_over_ranks(s2.elapsed_time(e2))
        e2e = {"value": replicas.whole_job_rate(op.units, K, world, e2e_ms), "unit": "rows/s",
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host_in),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in host_out),
               "api": "the binding call with pinned host buffers copied in and out by tp_mlp_copy_async, "
                      "synchronize per step"}
    sampler.stop()
    peaks, src = load_peaks()
    achieved = step_bytes / (launch_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": recorded_traffic(f"{op.family}:op", args.config),
                "kernel": op.kernel, "kernel_ms": launch_ms, "algorithmic_per_launch": step_bytes,
                "peak_source": f"hbm_gbs ({src})"}
    ms = elapsed_ms / K
    line = {"metric": op.metric, "value": replicas.whole_job_rate(op.units, K, world, elapsed_ms),
            "unit": "rows/s", "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": op.dtype,
            "data": "synthetic",
            "config": dict({"workload": op.workload, "parallelism": "replicas" if world > 1 else "single GPU",
                            "l2": (f"{copies} input copies rotated ({copies * step_bytes / 2 ** 20:.0f} MiB > L2)"
                                   if copies > 1 else "inputs larger than L2")}, **op.config),
            "step_hbm_gbs": step_bytes / (ms / 1e3) / 1e9, "roofline": roofline, "gpu_launches": K,
            "clocks": sampler.summary(), "e2e": e2e,
            "timer": "CUDA events around one replay of a CUDA graph holding the K launches",
            "python_call_us": api_ms * 1e3,
            "library_ops": {"ms": library_ms, "ops": op.library_ops, "algorithmic_bytes": op.library_bytes()}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, rows, tt = op.oracle_rate(10.0)
        line["cpu_baseline"] = {"value": v, "unit": "rows/s", "cores": 1, "kind": "oracle",
                                "sample": f"{rows} rows of this workload on one host core, {tt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    replicas.finish()
    return 0


def run_small_op_reference(args, op):
    """Reference arm of a small operator: its oracle on whole rows, bounded."""
    if int(os.environ.get("RANK", 0)) != 0:
        return 0
    budget = 150.0 / max(1, args.steps + args.warmup)
    done = []
    for i in range(args.warmup + args.steps):
        _, rows, tt = op.oracle_rate(budget)
        if i >= args.warmup:
            done.append((rows, tt))
    rows = sum(r for r, _ in done)
    tt = sum(t for _, t in done)
    value = rows / tt
    sample = f"each step: the oracle on whole rows for about {budget:.1f} s ({rows} rows in all)"
    line = {"impl": "reference", "metric": op.metric, "value": value, "unit": "rows/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict({"workload": op.workload, "parallelism": "host oracle"}, **op.config),
            "cpu_baseline": {"value": value, "unit": "rows/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# Workloads the default run times beside the headline, each on its own seeded
# inputs (name, tokens, tp): the rest of the metric -- decode at batch 32,
# prefill (TFLOP/s against the bf16 peak) and the TP x token sweep's
# memory-bound middle and compute-bound end.
EXTRA_CONFIGS = (("decode_bs32", None, None), ("prefill", None, 8), ("sweep", 16, 8), ("sweep", 128, 8),
                 ("sweep", 1024, 8))
EXTRA_MIN_TIMED_S = 0.25     # timed window of each extra workload (room for clock samples)
EXTRA_ORACLE_BUDGET_S = 4.0  # CPU-baseline budget of each extra workload (at least one call)
PHASE_NAMES = ["first projection + activation", "second projection + rank sum"]
# tc_fused: one persistent kernel runs both projections; the second projection's
# split tiles are added by a reduction kernel behind it.
FUSED_PHASE_NAMES = ["both projections (one persistent kernel)", "split-tile reduction of the second projection"]


def config_of(name, tokens=None, tp=None):
    ns = argparse.Namespace(config=name, tokens=tokens, tp=tp, d_model=None, d_ff=None)
    return resolve(ns)


class MlpRun:
    """One MLP workload on this GPU: seeded inputs, handle, weights packed once
    (or kept as shards), and the timing passes."""

    def __init__(self, c, plan="auto", splitk="auto", api="packed"):
        import torch

        from tensor_sharded_mlp_b200 import binding, inputs
        self.torch, self.binding, self.c, self.api = torch, binding, c, api
        T, d, f, tp, act, dt = c["tokens"], c["d_model"], c["d_ff"], c["tp"], c["act"], c["dtype"]
        self.p = inputs.generate(T, d, f, act, dt, c["seed"], c["init"])
        self.A, self.Bs = self.p.shards(tp)
        tdt = torch.bfloat16 if dt == "bf16" else torch.float32

        def up(a):
            return torch.from_numpy(a).cuda().to(tdt).contiguous()

        self.m = binding.TpMlp(d, f, tp, act, dt, max_tokens=T)
        self.m.set_plan(plan)
        self.m.set_splitk(splitk)
        Ad, Bd = [up(a) for a in self.A], [up(b) for b in self.Bs]
        # the one-off shard-layout pack, timed on its own (not part of a step)
        torch.cuda.synchronize()
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record()
        self.packed = self.m.pack(Ad, Bd)
        p1.record()
        p1.synchronize()
        self.pack_ms = p0.elapsed_time(p1)
        self.x = up(self.p.x)
        self.out = torch.empty(T, d, dtype=tdt, device="cuda")
        if api == "packed":
            del Ad, Bd
            self.fwd = lambda: self.m.forward_packed(self.x, self.packed, out=self.out)   # noqa: E731
        else:
            self.fwd = lambda: self.m.forward(self.x, Ad, Bd, out=self.out)              # noqa: E731
        torch.cuda.synchronize()

    def warm(self, W):
        for _ in range(W):
            self.fwd()
        self.torch.cuda.synchronize()
        self.nk = self.m.last_launches
        self.plan = self.m.last_plan

    def estimate_ms(self, n=5):
        torch = self.torch
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n):
            self.fwd()
        b.record()
        b.synchronize()
        return a.elapsed_time(b) / n

    TENSOR_PLANS = ("tc_wide", "tc_wide256", "tc_pair", "tc_pair2")

    def timed(self, K, barrier, kernel_events=False):
        """K clean steps back to back (each may overlap the previous one's tail
        through programmatic dependent launch), CUDA events on the launch stream,
        NVML clocks sampled over the window.  Returns (ms, clock summary, mean ms
        per phase or None).  kernel_events: the library also records events
        before, between and after its kernels inside this timed region -- for
        the tensor-bound tilings, whose millisecond kernels gain nothing from
        launch overlap, so each kernel is timed under the same clocks as the step."""
        torch = self.torch
        stream = torch.cuda.current_stream()
        ev = None
        if kernel_events:
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
            for row in ev:
                for e in row:
                    e.record(stream)
            torch.cuda.synchronize()
        sampler = ClockSampler(torch.cuda.current_device())
        sampler.start()
        time.sleep(0.1)
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        t0 = time.perf_counter()
        start.record(stream)
        for i in range(K):
            if ev is not None:
                self.binding.tp_mlp_set_profile_events(self.m.h, ev[i])
            self.fwd()
        end.record(stream)
        barrier()
        sampler.mark(t0, time.perf_counter())
        sampler.stop()
        phases = None
        if ev is not None:
            self.binding.tp_mlp_set_profile_events(self.m.h, None)
            phases = [statistics.fmean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K)) for j in range(2)]
        return start.elapsed_time(end), sampler.summary(), phases

    def phases(self, K, barrier):
        """The same K steps again with the library recording events before, between
        and after its kernels (kept apart from the timed pass: an event between two
        kernels disables their programmatic overlap).  Mean ms per phase."""
        torch = self.torch
        stream = torch.cuda.current_stream()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
        for row in ev:
            for e in row:
                e.record(stream)
        for i in range(K):
            self.binding.tp_mlp_set_profile_events(self.m.h, ev[i])
            self.fwd()
        self.binding.tp_mlp_set_profile_events(self.m.h, None)
        barrier()
        return [statistics.fmean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K)) for j in range(2)]

    def roofline(self, kern_ms, peaks, src, workload_key):
        """Roofline of the dominant kernel (largest share of the step): HBM bytes for
        the memory-bound tilings, FLOPs against the bf16 peak for the wide ones."""
        from tensor_sharded_mlp_b200 import counts
        c = self.c
        T, d, f, act, dt = c["tokens"], c["d_model"], c["d_ff"], c["act"], c["dtype"]
        j = int(np.argmax(kern_ms))
        fused = self.plan == "tc_fused"
        if fused:
            j = 0   # the kernel that streams both projections' weights
        extra = {}
        if self.plan in self.TENSOR_PLANS:
            bound, unit = "tensor", "TFLOP/s"
            work = counts.gemm1_flops(T, d, f, act) if j == 0 else counts.gemm2_flops(T, f, d)
            achieved = work / (kern_ms[j] / 1e3) / 1e12
            peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
            peak_note = f"bf16_tflops, burst ({src})"
            sus = peaks.get("bf16_tflops_sustained")
            if sus:
                extra = {"peak_sustained": sus, "frac_sustained": achieved / sus}
        else:
            bound, unit = "hbm", "GB/s"
            if fused:
                work = counts.gemm1_bytes(T, d, f, act, dt) + counts.gemm2_bytes(T, f, d, dt)
            else:
                work = counts.gemm1_bytes(T, d, f, act, dt) if j == 0 else counts.gemm2_bytes(T, f, d, dt)
            achieved = work / (kern_ms[j] / 1e3) / 1e9
            peak = peaks["hbm_gbs"]
            peak_note = f"hbm_gbs ({src})"
        kname = f"{self.plan}:{'first' if j == 0 else 'second'}" if not fused else "tc_fused:both"
        split = " (GEMM + split-tile reduction kernel)" if self.nk > 2 and self.plan == "tc_skinny" else ""
        r = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
             "traffic": recorded_traffic(kname, workload_key),
             "kernel": (FUSED_PHASE_NAMES if fused else PHASE_NAMES)[j] + split,
             "kernel_ms": kern_ms[j], "algorithmic_per_launch": work, "peak_source": peak_note,
             "kernel_ms_all": kern_ms,
             "kernel_timer": ("CUDA events around each kernel inside the timed region"
                              if self.plan in self.TENSOR_PLANS else
                              "CUDA events around each kernel in a second pass of the same steps (an event "
                              "between two kernels would stop their launch overlap in the timed region)")}
        r.update(extra)
        return r

    def step_rates(self, ms):
        from tensor_sharded_mlp_b200 import counts
        c = self.c
        T, d, f, act, dt = c["tokens"], c["d_model"], c["d_ff"], c["act"], c["dtype"]
        step_bytes = counts.algorithmic_bytes(T, d, f, d, act, dt)
        return {"step_hbm_gbs": step_bytes / (ms / 1e3) / 1e9,
                "step_tflops": counts.forward_flops(T, d, f, d, act) / (ms / 1e3) / 1e12}, step_bytes


def measure_extra(name, tokens, tp, args, peaks, src, barrier, cpu):
    """One extra workload of the metric: its own inputs, warm-up, a timed window of
    at least EXTRA_MIN_TIMED_S, per-phase kernel times, roofline, clocks, and a
    bounded CPU baseline of the oracle."""
    import torch

    from tensor_sharded_mlp_b200 import counts
    c = config_of(name, tokens, tp)
    t_gen = time.perf_counter()
    run = MlpRun(c)
    t_gen = time.perf_counter() - t_gen
    W = max(3, args.warmup)
    run.warm(W)
    est = run.estimate_ms()
    K = max(args.steps, int(np.ceil(EXTRA_MIN_TIMED_S * 1e3 / max(est, 1e-3))))
    ms_total, clocks, kern_ms = run.timed(K, barrier, kernel_events=run.plan in MlpRun.TENSOR_PLANS)
    if kern_ms is None:
        kern_ms = run.phases(min(K, 200), barrier)
    ms = ms_total / K
    rates, step_bytes = run.step_rates(ms)
    key = name if tokens is None else f"{name}_T{tokens}"
    e = {"workload": c["workload"], "tokens": c["tokens"], "tp": c["tp"], "plan": run.plan, "steps": K,
         "warmup": W, "ms_per_step": ms, "value": c["tokens"] * K / (ms_total / 1e3), "unit": "tokens/s",
         "roofline": run.roofline(kern_ms, peaks, src, key), "clocks": clocks, "gpu_launches": K * run.nk,
         "timer": "CUDA events on the launch stream around the K steps",
         "l2": "inputs larger than L2: every step re-reads %.2f GB of weights" % (
             counts.weight_bytes(c["d_model"], c["d_ff"], c["d_model"], c["act"], c["dtype"]) / 1e9),
         "pack_ms": run.pack_ms, "host_setup_s": t_gen}
    e.update(rates)
    if cpu:
        sample = c.get("sample_rows", 256) if c["tokens"] > 256 else None
        e["cpu_baseline"] = oracle_baseline(run.p, run.A, run.Bs, c["act"], budget_s=EXTRA_ORACLE_BUDGET_S,
                                            max_calls=20, sample_rows=sample, one_core=False)
    del run
    torch.cuda.empty_cache()
    return key, e


XGPU_METRIC = "cross-GPU tensor-parallel MLP step (one rank per GPU): tokens/s, fused one-shot all-reduce vs NCCL"


def run_xgpu(args):
    """--config xgpu_decode_bs32: the decode batch-32 MLP (bf16 SwiGLU, d 8192,
    f 28672) with tp = the number of ranks, one rank per GPU.  Times the fused
    step (tp_mlp_xgpu_forward: the one-shot all-reduce inside the second
    projection) against the unfused one (each rank's fp32 partial from the
    library, then the process group's NCCL all_reduce), max over ranks.  The
    weights are random on the device (seeded per rank); correctness is the tests'
    business.  The whole job processes T tokens per step: strong scaling."""
    import torch

    from tensor_sharded_mlp_b200 import replicas, xgpu
    rank, world, local = replicas.rank_env()
    torch.cuda.set_device(local)
    replicas.init("nccl", torch.device("cuda", local), timeout_s=120)
    d, f, T = 8192, 28672, args.tokens or 32
    tp = world
    fs = f // tp
    g = torch.Generator(device="cuda")
    g.manual_seed(1000 + rank)
    A_r = (torch.randn(d, 2 * fs, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
    B_r = (torch.randn(fs, d, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
    g.manual_seed(7)                                   # the same tokens on every rank
    x = torch.randn(T, d, device="cuda", generator=g).to(torch.bfloat16)
    fused = xgpu.CrossGpuMlp(d, f, tp, "swiglu", T, rank, A_r, B_r)
    unfused = xgpu.LibraryAllReduceMlp(d, f, tp, "swiglu", T, A_r, B_r)
    out = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    K, W = args.steps, max(3, args.warmup)

    def timed(fn):
        for _ in range(W):
            fn()
        replicas.barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(K):
            fn()
        b.record()
        b.synchronize()
        replicas.barrier()
        return replicas.max_over_ranks(a.elapsed_time(b))

    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    ms_fused = timed(lambda: fused.forward(x, out))
    ms_nccl = timed(lambda: unfused.forward(x))
    sampler.stop()
    agree = float((fused.forward(x, out).float() - unfused.forward(x).float()).abs().max())
    torch.cuda.synchronize()
    fused.close()
    if rank == 0:
        line = {"metric": XGPU_METRIC, "value": T * K / (ms_fused / 1e3), "unit": "tokens/s", "n_gpus": world,
                "steps": K, "warmup": W, "ms_per_step": ms_fused / K, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": f"xgpu_decode_bs32: bf16 SwiGLU MLP, tokens={T}, d_model={d}, d_ff={f}, "
                                       f"tp={tp} (one rank per GPU), random weights N(0,0.02^2)",
                           "tokens": T, "d_model": d, "d_ff": f, "tp": tp, "parallelism": f"tp{tp}"},
                "nccl_allreduce_arm": {"ms_per_step": ms_nccl / K, "value": T * K / (ms_nccl / 1e3),
                                       "unit": "tokens/s",
                                       "what": "library fp32 partial per rank + torch.distributed all_reduce"},
                "max_abs_difference_between_arms": agree, "gpu_launches": K * 2, "clocks": sampler.summary(),
                "note": "n_gpus=1 has no exchange partner (tp 1)" if world == 1 else ""}
        print(json.dumps(line), flush=True)
    replicas.finish()
    return 0


def main():
    args = parse()
    if args.config == "xgpu_decode_bs32":
        if args.impl == "reference":
            if int(os.environ.get("RANK", 0)) == 0:
                print(json.dumps({"impl": "reference", "unavailable": "the cross-GPU mode has no oracle arm; "
                                  "its correctness is in tests/test_gpu_xgpu.py"}), flush=True)
            return 0
        return run_xgpu(args)
    op = small_op(args)
    if op is not None:
        return run_small_op_reference(args, op) if args.impl == "reference" else run_small_op(args, op)
    if args.impl == "reference":
        return run_reference(args)

    import torch

    from tensor_sharded_mlp_b200 import binding, counts, replicas

    rank, world, local = replicas.rank_env()
    torch.cuda.set_device(local)
    replicas.init("nccl", torch.device("cuda", local))
    c = resolve(args)
    T, d, f, tp, act, dt = c["tokens"], c["d_model"], c["d_ff"], c["tp"], c["act"], c["dtype"]
    run = MlpRun(c, args.plan, args.splitk, args.api)
    m, packed, x, out, fwd = run.m, run.packed, run.x, run.out, run.fwd

    def barrier():
        replicas.barrier()
        torch.cuda.synchronize()

    K, W = args.steps, max(3, args.warmup)
    run.warm(W)
    nk, plan = run.nk, run.plan
    elapsed_ms, clocks, kern_ms = run.timed(K, barrier, kernel_events=plan in MlpRun.TENSOR_PLANS)
    if kern_ms is None:
        kern_ms = run.phases(K, barrier)
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
        s2.record(torch.cuda.current_stream())
        for _ in range(K):
            step()                    # replay + wait for the result on the host
        e2.record(torch.cuda.current_stream())
        e2.synchronize()
        e2e_ms = replicas.max_over_ranks(s2.elapsed_time(e2))
        ref_out = out.cpu()
        e2e_ok = bool(torch.equal(step.out_host, ref_out))
        e2e = {"value": replicas.whole_job_rate(T, K, world, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": step.x_host.numel() * step.x_host.element_size(),
               "d2h_bytes_per_step": step.out_host.numel() * step.out_host.element_size(),
               "api": "binding.GraphStep (CUDA graph: tp_mlp_copy_async H2D x, tp_mlp_forward_packed, "
                      "tp_mlp_copy_async D2H out; synchronize)",
               "timer": "CUDA events on the replay stream around K steps, host waits included",
               "matches_device_result": e2e_ok}
        del step

    value = replicas.whole_job_rate(T, K, world, elapsed_ms)
    peaks, src = load_peaks()
    ms = elapsed_ms / K
    rates, step_bytes = run.step_rates(ms)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": dt, "data": "synthetic",
            "config": {"workload": c["workload"], "tokens": T, "d_model": d, "d_ff": f, "tp": tp, "act": act,
                       "plan": plan, "splitk": args.splitk, "api": args.api,
                       "parallelism": "replicas" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2: every step re-reads %.2f GB of weights" % (step_bytes / 1e9)},
            "roofline": run.roofline(kern_ms, peaks, src, args.config), "gpu_launches": K * nk,
            "clocks": clocks, "e2e": e2e, "graph_step": graph_steps,
            "pack": {"ms": run.pack_ms, "note": "one-off shard-layout pack before timing (first call, includes "
                                               "the packer's launch set-up); reads and writes every weight once",
                     "GBs": 2 * counts.weight_bytes(d, f, d, act, dt) / (run.pack_ms / 1e3) / 1e9}}
    line.update(rates)
    cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    if cpu:
        line["cpu_baseline"] = oracle_baseline(run.p, run.A, run.Bs, act)
    del run, m, packed, x, out, fwd
    torch.cuda.empty_cache()
    # the rest of the metric, in the same run (one GPU only: each workload is
    # generated on the host, and a replica per rank would multiply that)
    if extra_configs_wanted(args) and world == 1:
        line["configs"] = {}
        for name, tk, tpx in EXTRA_CONFIGS:
            key, e = measure_extra(name, tk, tpx, args, peaks, src, barrier, cpu)
            line["configs"][key] = e
    if rank == 0:
        print(json.dumps(line), flush=True)
    replicas.finish()
    return 0


def extra_configs_wanted(args):
    if args.configs == "none":
        return False
    if args.configs == "all":
        return True
    # auto: the default invocation (the headline workload, nothing overridden)
    return (args.config == "decode_bs1" and args.tokens is None and args.tp is None and args.plan == "auto"
            and args.api == "packed" and args.splitk == "auto" and args.d_model is None and args.d_ff is None)


if __name__ == "__main__":
    sys.exit(main())
