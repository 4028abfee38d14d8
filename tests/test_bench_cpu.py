"""Host logic of bench.py that decides what a run measures (CPU only).

The default invocation -- the workload the metric is quoted on, nothing
overridden -- also times the rest of the metric (decode batch 32, prefill and
the sweep points) in a "configs" block; any override, or --configs none,
times one workload only (the ncu harness relies on that).
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _args(*argv):
    old = sys.argv
    sys.argv = ["bench.py", *argv]
    try:
        return bench.parse()
    finally:
        sys.argv = old


def test_default_invocation_times_every_config():
    assert bench.extra_configs_wanted(_args())
    assert bench.extra_configs_wanted(_args("--steps", "20", "--warmup", "5", "--gpus", "1"))


def test_overrides_time_one_workload():
    for argv in (["--config", "decode_bs32"], ["--tokens", "2"], ["--tp", "4"], ["--plan", "gemv"],
                 ["--api", "shard"], ["--splitk", "separate"], ["--d-model", "1024"], ["--configs", "none"]):
        assert not bench.extra_configs_wanted(_args(*argv)), argv
    assert bench.extra_configs_wanted(_args("--config", "decode_bs32", "--configs", "all"))


def test_extra_configs_are_the_metric_workloads():
    names = [(n, t, p) for n, t, p in bench.EXTRA_CONFIGS]
    assert ("decode_bs32", None, None) in names and ("prefill", None, 8) in names
    assert {t for n, t, _ in names if n == "sweep"} == {16, 128, 1024}
    for n, t, p in names:
        c = bench.config_of(n, t, p)
        assert c["workload"].startswith(n) and c["tokens"] >= 1 and c["tp"] in (1, 2, 4, 8)
    assert bench.config_of("prefill", None, 8)["sample_rows"] == 256
