"""The N > 1 path on CPU: world-size-2 process groups over gloo.

bench.py runs one independent replica per GPU; its multi-rank logic is the
host code in tensor_sharded_mlp_b200.replicas (barriers, max over ranks,
whole-job rate).  Here two gloo ranks exercise that code, and torchrun runs the
reference arm of bench.py with two ranks, of which only rank 0 may print.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from tensor_sharded_mlp_b200 import replicas
    replicas.init("gloo", timeout_s=60)
    r, w, lr = replicas.rank_env()
    replicas.barrier()
    mine = 10.0 + 5.0 * rank            # rank 1 is the slower one
    worst = replicas.max_over_ranks(mine)
    rate = replicas.whole_job_rate(units_per_rank_step=32, steps=100, world=w, max_ms=worst)
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"rank": r, "world": w, "local": lr, "worst": worst, "rate": rate}, f)
    replicas.finish()


def test_two_gloo_ranks_agree_on_the_slowest_time(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"r{i}.json")) for i in range(2)]
    assert [r["rank"] for r in res] == [0, 1] and all(r["world"] == 2 for r in res)
    assert all(r["worst"] == 15.0 for r in res)               # max over ranks, on every rank
    assert all(r["rate"] == pytest.approx(2 * 32 * 100 / 0.015) for r in res)


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    from tensor_sharded_mlp_b200 import replicas
    assert replicas.max_over_ranks(3.5) == 3.5
    assert replicas.whole_job_rate(1, 10, 1, 2.0) == pytest.approx(5000.0)
    with pytest.raises(ValueError):
        replicas.whole_job_rate(1, 1, 1, 0.0)


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--config", "tiny", "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def _worker_one_leaves(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import time
    from tensor_sharded_mlp_b200 import replicas
    replicas.init("gloo", timeout_s=5)
    replicas.barrier()                     # both ranks are up
    if rank == 1:
        return                             # rank 1 leaves between steps, with nothing in flight
    t0 = time.time()
    outcome = "no error"
    try:
        replicas.max_over_ranks(1.0)       # the next collective must fail, not hang
    except Exception as e:                 # gloo reports the lost peer or the timeout
        outcome = type(e).__name__
    with open(os.path.join(out_dir, "survivor.json"), "w") as f:
        json.dump({"outcome": outcome, "seconds": time.time() - t0}, f)


def test_a_rank_that_leaves_is_detected_by_the_next_collective(tmp_path):
    port = _free_port()
    mp.start_processes(_worker_one_leaves, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn",
                       join=True)
    r = json.load(open(tmp_path / "survivor.json"))
    assert r["outcome"] != "no error"
    assert r["seconds"] < 60
