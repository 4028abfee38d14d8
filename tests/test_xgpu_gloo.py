"""Host side of tensor parallelism across GPUs, on CPU with gloo ranks.

The kernels need GPUs; what runs here is the host logic around them: the
exchange of the ranks' buffer handles over a process group, the comparison
arm's all_reduce of the ranks' partials (checked against the
oracle: the rank sum equals the unsharded MLP), and a rank that leaves before
the exchange, which the others must notice instead of hanging.
"""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)


def _worker_exchange(rank, world, port, out_dir):
    _env(rank, world, port)
    import torch
    import torch.distributed as dist
    from tensor_sharded_mlp_b200 import xgpu
    dist.init_process_group("gloo", rank=rank, world_size=world)
    mine = (bytes([rank + 1]) * 64, 4096 * rank + 16)
    handles = xgpu.exchange_handles(mine)
    opened = []

    def fake_open(h, off):                 # stands in for CUDA IPC: records what it is asked to map
        opened.append((h[0], off))
        return 1_000_000 * (h[0]) + off
    ptrs = xgpu.open_peers(handles, rank, own_ptr=777, opener=fake_open)
    # the comparison arm's exchange: each rank's oracle partial, summed by the group
    import oracle
    from tensor_sharded_mlp_b200 import inputs
    p = inputs.generate(3, 32, 64, "swiglu", "f32", seed=5, init="fan_in")
    A, B = p.shards(world)
    z = torch.from_numpy(oracle.tp_mlp_sharded(p.x, [A[rank]], [B[rank]], "swiglu").astype(np.float32))
    xgpu.allreduce_partial(z)
    ref = oracle.tp_mlp_unsharded(p.x, p.gate, p.b, "swiglu", a_up=p.up)
    err = float(np.max(np.abs(z.numpy() - ref)) / np.max(np.abs(ref)))
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"handles": [[h[0][0], h[1]] for h in handles], "ptrs": ptrs, "opened": opened, "err": err}, f)
    dist.destroy_process_group()


def test_exchange_and_library_allreduce_on_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_worker_exchange, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"r{i}.json")) for i in range(2)]
    for rank, r in enumerate(res):
        assert r["handles"] == [[1, 16], [2, 4112]]             # every rank's handle, in rank order
        peer = 1 - rank
        assert r["opened"] == [[peer + 1, 4096 * peer + 16]]     # only the peer is mapped, at its offset
        assert r["ptrs"][rank] == 777                            # our own buffer is used as it is
        assert r["ptrs"][peer] == 1_000_000 * (peer + 1) + 4096 * peer + 16
        assert r["err"] <= 1e-5                                   # rank sum == unsharded MLP (fp32 sum)


def _worker_leaves(rank, world, port, out_dir, when):
    _env(rank, world, port)
    import datetime
    import time
    import torch
    import torch.distributed as dist
    from tensor_sharded_mlp_b200 import xgpu
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    dist.barrier()
    if when == "before_exchange" and rank == 1:
        return                              # leaves before the handle exchange, nothing in flight
    steps_done = 0
    if when == "between_steps":
        xgpu.exchange_handles((bytes([rank + 1]) * 64, 0))
        for _ in range(2):                  # two steps of the comparison arm's exchange
            xgpu.allreduce_partial(torch.ones(4, 8))
            steps_done += 1
        if rank == 1:
            return                          # leaves between steps, nothing in flight
    t0 = time.time()
    outcome = "no error"
    try:
        if when == "before_exchange":
            xgpu.exchange_handles((bytes(64), 0))
        else:
            xgpu.allreduce_partial(torch.ones(4, 8))
    except Exception as e:
        outcome = type(e).__name__
    with open(os.path.join(out_dir, "survivor.json"), "w") as f:
        json.dump({"outcome": outcome, "seconds": time.time() - t0, "steps_done": steps_done}, f)


@pytest.mark.parametrize("when", ["before_exchange", "between_steps"])
def test_a_rank_that_leaves_is_detected(tmp_path, when):
    port = _free_port()
    mp.start_processes(_worker_leaves, args=(2, port, str(tmp_path), when), nprocs=2, start_method="spawn",
                       join=True)
    r = json.load(open(tmp_path / "survivor.json"))
    assert r["outcome"] != "no error"
    assert r["seconds"] < 60
    assert r["steps_done"] == (2 if when == "between_steps" else 0)
