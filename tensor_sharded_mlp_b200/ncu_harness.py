"""ncu harness: capture commands for the library's kernels and summaries of the results.

Captures run on a machine with the GPU; summaries are made anywhere ncu can
open the report (``ncu -i``).  Three kinds of capture, all with
``--clock-control none`` (never lock the GPU clocks):

* launch list  -- ``gpu__time_duration.sum`` only (one pass), any workload size:
      python -m tensor_sharded_mlp_b200.ncu_harness list-cmd --config decode_bs1
* full set     -- ``--set full`` on ONE kernel (``-k``), 1 launch, on a reduced
  workload that still exceeds L2 but holds at most a few GB on the device:
      python -m tensor_sharded_mlp_b200.ncu_harness full-cmd --kernel gemv_kernel --config decode_bs1 \
          --d-model 4096 --d-ff 14336
* summaries    -- turn a launch-list CSV or a full report into the markdown kept
  under profiles/, and record DRAM bytes per launch (scaled to the full workload
  by the units processed) in profiles/dram_traffic.json for bench.py:
      python -m tensor_sharded_mlp_b200.ncu_harness summarize-list launches.csv --title ... --out ...
      python -m tensor_sharded_mlp_b200.ncu_harness summarize-full prof.ncu-rep --title ... --out ... \
          [--traffic-key plan:first|config --scale 4.0 --launch 0]

Each summary records the command that produced it.
"""
from __future__ import annotations

import argparse
import collections
import csv
import io
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

FULL_METRICS = [
    "gpu__time_duration.sum",
    "dram__bytes_read.sum",
    "dram__bytes_write.sum",
    "gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed",
    "dram__throughput.avg.pct_of_peak_sustained_elapsed",
    "sm__throughput.avg.pct_of_peak_sustained_elapsed",
    "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed",
    "sm__pipe_tensor_op_hmma_cycles_active.avg.pct_of_peak_sustained_elapsed",
    "sm__inst_executed_pipe_tc.avg.pct_of_peak_sustained_elapsed",
    "sm__warps_active.avg.pct_of_peak_sustained_active",
    "launch__registers_per_thread",
    "launch__grid_size",
    "launch__block_size",
    "launch__shared_mem_per_block_dynamic",
    "launch__waves_per_multiprocessor",
    "launch__occupancy_limit_registers",
    "launch__occupancy_limit_shared_mem",
    "lts__t_bytes.sum",
    "lts__t_sector_hit_rate.pct",
    "smsp__average_warps_issue_stalled_long_scoreboard_per_issue_active.ratio",
    "smsp__issue_active.avg.pct_of_peak_sustained_active",
    "sm__cycles_elapsed.avg.per_second",
    "dram__cycles_elapsed.avg.per_second",
]


def bench_cmd(config: str, extra: list[str]) -> str:
    return " ".join(["python", "bench.py", "--config", config, "--steps", "2", "--warmup", "3",
                     "--no-e2e", "--no-cpu-baseline", "--no-graph", "--configs", "none"] + extra)


def list_cmd(a) -> str:
    return (f"ncu --metrics gpu__time_duration.sum --clock-control none --csv "
            f"--log-file {a.out_dir}/launches_{a.config}.csv {bench_cmd(a.config, a.extra)}")


def full_cmd(a) -> str:
    return (f"ncu --set full --clock-control none -k regex:{a.kernel} -s 3 -c 1 "
            f"-o {a.out_dir}/prof_{a.kernel}_{a.config} {bench_cmd(a.config, a.extra)}")


def _read_csv_rows(text: str):
    lines = [l for l in text.splitlines() if l.startswith('"')]
    return list(csv.reader(io.StringIO("\n".join(lines))))


def _to_ns(v: float, unit: str) -> float:
    return v * {"nsecond": 1, "usecond": 1e3, "msecond": 1e6, "second": 1e9}.get(unit, 1)


def summarize_list(path: str, title: str, cmd: str) -> str:
    rows = _read_csv_rows(open(path).read())
    h = rows[0]
    ki, vi, ui = h.index("Kernel Name"), h.index("Metric Value"), h.index("Metric Unit")
    agg = collections.OrderedDict()
    each = collections.defaultdict(list)
    for r in rows[1:]:
        if len(r) <= vi or r[h.index("Metric Name")] != "gpu__time_duration.sum":
            continue
        name = r[ki].split("(")[0].replace("void ", "").replace("tpmlp::", "").replace("<unnamed>::", "")
        a = agg.setdefault(name, [0, 0.0])
        a[0] += 1
        t = _to_ns(float(r[vi].replace(",", "")), r[ui])
        a[1] += t
        each[name].append(t)
    total = sum(a[1] for a in agg.values())
    out = [f"# {title}", "", "Launch list from one ncu pass (`gpu__time_duration.sum` only).  Per-launch",
           "times here are serialised and cold-cache: compare shares, not absolute times.", "",
           "Command:", "", "```", cmd, "```", "",
           "| kernel | launches | total µs | mean µs | share |", "|---|---:|---:|---:|---:|"]
    for k, (n, t) in sorted(agg.items(), key=lambda x: -x[1][1]):
        out.append(f"| `{k}` | {n} | {t / 1e3:.1f} | {t / n / 1e3:.1f} | {100 * t / total:.1f}% |")
    # the kernels a forward launches (not the one-off pack or torch's input copies)
    step = {k: v for k, v in agg.items() if k.startswith(STEP_KERNELS)}
    st = sum(v[1] for v in step.values())
    if step and st > 0:
        out += ["", "Shares among the forward's own kernels (the timed region launches only these):", "",
                "| kernel | launches | total µs | mean µs | share of the forward |", "|---|---:|---:|---:|---:|"]
        for k, (n, t) in sorted(step.items(), key=lambda x: -x[1][1]):
            out.append(f"| `{k}` | {n} | {t / 1e3:.1f} | {t / n / 1e3:.1f} | {100 * t / st:.1f}% |")
        alt = {k: v for k, v in each.items() if k in step and len(v) % 2 == 0 and len(v) >= 2}
        if alt:
            out += ["", "A forward launches its first projection, then its second; where one kernel",
                    "serves both, its launches alternate:", "",
                    "| kernel | mean µs, 1st, 3rd, ... launch | mean µs, 2nd, 4th, ... launch |", "|---|---:|---:|"]
            for k, v in alt.items():
                out.append(f"| `{k}` | {sum(v[0::2]) / len(v[0::2]) / 1e3:.1f} | {sum(v[1::2]) / len(v[1::2]) / 1e3:.1f} |")
    return "\n".join(out) + "\n"


STEP_KERNELS = ("gemv_kernel", "tc_fused_kernel", "tc_skinny_kernel", "skinny_reduce_kernel", "tc_wide_kernel", "tc_pair_kernel",
                "simt_", "allreduce_norm_kernel", "attn_merge_kernel", "unnamed>::tc_", "unnamed>::skinny",
                "unnamed>::gemv")


def _raw(report: str):
    txt = subprocess.run(["ncu", "-i", report, "--page", "raw", "--csv"], capture_output=True, text=True,
                         check=True).stdout
    rows = _read_csv_rows(txt)
    return rows[0], rows[1], rows[2:]


def summarize_full(report: str, title: str, cmd: str, traffic_key=None, scale=1.0, note="", launch=0):
    h, units, rows = _raw(report)
    idx = {n: i for i, n in enumerate(h)}
    out = [f"# {title}", "", "One `--set full` capture (clocks not locked).  " + note, "", "Command:", "", "```",
           cmd, "```", ""]
    traffic = None
    for li, r in enumerate(rows):
        kname = r[idx["Kernel Name"]].split("(")[0]
        out += [f"## `{kname}`", "", "| metric | value | unit |", "|---|---:|---|"]
        for m in FULL_METRICS:
            if m in idx and r[idx[m]] != "":
                out.append(f"| `{m}` | {r[idx[m]]} | {units[idx[m]]} |")
        try:
            def val(m):
                v = float(r[idx[m]].replace(",", ""))
                u = units[idx[m]]
                return v * {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}.get(u, 1)
            rd, wr = val("dram__bytes_read.sum"), val("dram__bytes_write.sum")
            if li == launch:
                traffic = (rd + wr) * scale
            out += ["", f"DRAM traffic per launch: {(rd + wr) / 1e6:.1f} MB"
                    + (f"; scaled ×{scale:g} to the full workload: {(rd + wr) * scale / 1e6:.1f} MB"
                       if scale != 1 else "")]
        except (KeyError, ValueError):
            pass
        out.append("")
    if traffic_key and traffic is not None:
        path = os.path.join(ROOT, "profiles", "dram_traffic.json")
        rec = json.load(open(path)) if os.path.exists(path) else {}
        from tensor_sharded_mlp_b200.counts import kernel_source_hash
        rec[traffic_key] = {"bytes_per_launch": traffic, "report": os.path.basename(report), "scale": scale,
                            "source_hash": kernel_source_hash(traffic_key.split(":")[0])}
        with open(path, "w") as f:
            json.dump(rec, f, indent=1, sort_keys=True)
    return "\n".join(out)


def main(argv=None):
    ap = argparse.ArgumentParser()
    sub = ap.add_subparsers(dest="cmd", required=True)
    for n in ("list-cmd", "full-cmd"):
        p = sub.add_parser(n)
        p.add_argument("--config", default="decode_bs1")
        p.add_argument("--kernel", default="gemv_kernel")
        p.add_argument("--out-dir", default="ncu_out", help="where ncu writes the CSV or report")
        p.add_argument("extra", nargs=argparse.REMAINDER)
    p = sub.add_parser("summarize-list")
    p.add_argument("csv")
    p.add_argument("--title", required=True)
    p.add_argument("--command", required=True)
    p.add_argument("--out", required=True)
    p = sub.add_parser("summarize-full")
    p.add_argument("report")
    p.add_argument("--title", required=True)
    p.add_argument("--command", required=True)
    p.add_argument("--out", required=True)
    p.add_argument("--traffic-key", default=None)
    p.add_argument("--scale", type=float, default=1.0)
    p.add_argument("--note", default="")
    p.add_argument("--launch", type=int, default=0, help="which captured launch the traffic key takes")
    a = ap.parse_args(argv)
    if a.cmd == "list-cmd":
        print(list_cmd(a))
    elif a.cmd == "full-cmd":
        print(full_cmd(a))
    elif a.cmd == "summarize-list":
        open(a.out, "w").write(summarize_list(a.csv, a.title, a.command))
    else:
        open(a.out, "w").write(summarize_full(a.report, a.title, a.command, a.traffic_key, a.scale, a.note,
                                              a.launch))
    return 0


if __name__ == "__main__":
    sys.exit(main())
