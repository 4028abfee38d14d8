"""Host logic for running the MLP as independent replicas, one process per GPU.

Every rank serves its own batch with its own copy of the weights: no data
moves between ranks ("7.4 推理侧并行" §7.4.1: with no gradients the
data-parallel dimension becomes pure replication with zero communication;
"LLM 推理并行化：先找瓶颈，再决定怎么切" §三 1) 数据并行).  The only collectives
are on the host side of the measurement: a barrier around the timed region and
the max over ranks of the measured time.
"""
from __future__ import annotations

import datetime
import os
from typing import Tuple

import torch
import torch.distributed as dist


def rank_env() -> Tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment (defaults: single process)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def init(backend: str, device=None, timeout_s: float = 300.0) -> None:
    """Join the process group when there is more than one rank."""
    _, world, _ = rank_env()
    if world > 1 and not dist.is_initialized():
        kw = {"device_id": device} if (backend == "nccl" and device is not None) else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def barrier() -> None:
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(value: float) -> float:
    """The largest value any rank measured (every rank gets it)."""
    if not (dist.is_initialized() and dist.get_world_size() > 1):
        return float(value)
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Units processed by all ranks per second, timed by the slowest rank."""
    if max_ms <= 0:
        raise ValueError("non-positive time")
    return world * units_per_rank_step * steps / (max_ms / 1e3)


def finish() -> None:
    if dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
