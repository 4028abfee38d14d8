"""Tensor parallelism across GPUs, one process per GPU: the host side.

Rank r holds only its shards A_r and B_r on GPU r ("LLM 推理并行化" §三 2);
"大模型推理系统揭秘（07）" §1.2.2-§1.2.3).  The sum of the ranks' partials
Z_r = act(x A_r) B_r is an all-reduce between GPUs, one per MLP.  The library
fuses it into the second projection as the one-shot all-reduce of
"7.4 推理侧并行" §7.4.2, optimisation 2 (tp_mlp_xgpu_forward): every rank stores
its bf16 partial tiles straight into every rank's exchange buffer and adds the
ranks' tiles itself.  This module does the plumbing around that call:

  * each rank allocates its exchange buffer on its own GPU (torch) and the
    ranks swap CUDA IPC handles over the process group, so every rank holds
    every buffer's address;
  * the comparison arm: each rank's fp32 partial from the library, summed with
    the process group's own all_reduce (NCCL on GPUs).

The sequence-parallel form (§7.4.2, optimisation 3: all-gather before the
first projection, reduce-scatter after the second) uses the same buffers
(tp_mlp_xgpu_sp_forward, forward_sp below).

The data path runs in the library's kernels; nothing here does arithmetic on
the MLP except the comparison arm's library all_reduce.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

Handle = Tuple[bytes, int]   # (64-byte CUDA IPC handle, offset of the buffer in its allocation)


def exchange_handles(local: Handle, group=None) -> List[Handle]:
    """Every rank's (handle, offset), in rank order, on every rank (a single
    process without a process group has only its own)."""
    if not dist.is_initialized():
        return [(bytes(local[0]), int(local[1]))]
    world = dist.get_world_size(group)
    out: List[Optional[Handle]] = [None] * world
    dist.all_gather_object(out, (bytes(local[0]), int(local[1])), group=group)
    for r, h in enumerate(out):
        if h is None or len(h[0]) != 64:
            raise RuntimeError(f"rank {r} sent no valid exchange-buffer handle")
    return [(h[0], h[1]) for h in out]


def open_peers(handles: Sequence[Handle], rank: int, own_ptr: int,
               opener: Optional[Callable[[bytes, int], int]] = None) -> List[int]:
    """Addresses of every rank's exchange buffer in this process: our own
    buffer as it is, the peers' through IPC (opener(handle, offset))."""
    if opener is None:
        from tensor_sharded_mlp_b200 import binding
        opener = binding.tp_mlp_ipc_open_handle
    return [own_ptr if r == rank else int(opener(h, off)) for r, (h, off) in enumerate(handles)]


class CrossGpuMlp:
    """One rank of the cross-GPU tensor-parallel MLP (bf16, 1..128 tokens).

        mlp = CrossGpuMlp(d_model, d_ff, tp, "swiglu", max_tokens, rank, A_r, B_r)
        out = mlp.forward(x)          # the full sum over ranks, on every rank

    Collective: every rank must construct it (the handle exchange) and then
    make the same forward calls with the same token counts."""

    def __init__(self, d_model: int, d_ff: int, tp: int, act: str, max_tokens: int, rank: int,
                 A_r: torch.Tensor, B_r: torch.Tensor, group=None, d_out: Optional[int] = None):
        from tensor_sharded_mlp_b200 import binding
        self.b = binding
        self.rank, self.tp = rank, tp
        self.A_r, self.B_r = A_r, B_r
        self.mlp = binding.TpMlp(d_model, d_ff, tp, act, "bf16", max_tokens=max_tokens, d_out=d_out)
        nbytes = binding.tp_mlp_xgpu_comm_bytes(self.mlp.h)
        self.comm = torch.zeros(nbytes, dtype=torch.uint8, device=self.mlp.device)
        torch.cuda.synchronize()
        handles = exchange_handles(binding.tp_mlp_ipc_get_handle(self.comm), group)
        self.ptrs = open_peers(handles, rank, self.comm.data_ptr())
        self._opened = [(self.ptrs[r], handles[r][1]) for r in range(tp) if r != rank]

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        if out is None:
            out = torch.empty(x.shape[0], self.mlp.d_out, dtype=torch.bfloat16, device=x.device)
        self.b.tp_mlp_xgpu_forward(self.mlp.h, self.rank, x, [self.A_r], [self.B_r], self.ptrs, [out], stream)
        return out

    def forward_sp(self, x_rows: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """Sequence-parallel form: x_rows are this rank's tokens / tp rows; returns
        this rank's rows of the output (all-gather and reduce-scatter fused)."""
        if out is None:
            out = torch.empty(x_rows.shape[0], self.mlp.d_out, dtype=torch.bfloat16, device=x_rows.device)
        self.b.tp_mlp_xgpu_sp_forward(self.mlp.h, self.rank, [x_rows], [self.A_r], [self.B_r], self.ptrs, [out],
                                      stream)
        return out

    def close(self):
        for ptr, off in self._opened:
            self.b.tp_mlp_ipc_close_handle(ptr, off)
        self._opened = []


def allreduce_partial(z: torch.Tensor, group=None) -> torch.Tensor:
    """The comparison arm's exchange: the process group's all_reduce (sum) of
    this rank's partial, in place (NCCL for CUDA tensors, gloo on the CPU)."""
    if dist.is_initialized():
        dist.all_reduce(z, op=dist.ReduceOp.SUM, group=group)
    return z


class LibraryAllReduceMlp:
    """Comparison arm: rank r's fp32 partial Z_r from the library (a one-rank
    handle over its own shards), then the process group's all_reduce, then the
    cast to bf16 -- the unfused step the pages start from."""

    def __init__(self, d_model: int, d_ff: int, tp: int, act: str, max_tokens: int, A_r: torch.Tensor,
                 B_r: torch.Tensor, group=None, d_out: Optional[int] = None):
        from tensor_sharded_mlp_b200 import binding
        self.group = group
        self.A_r, self.B_r = A_r, B_r
        self.one = binding.TpMlp(d_model, d_ff // tp, 1, act, "bf16", max_tokens=max_tokens, d_out=d_out)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        z = self.one.partials(x, [self.A_r], [self.B_r])[0]
        return allreduce_partial(z, self.group).to(torch.bfloat16)


class EmulatedRanks:
    """Every rank of the cross-GPU step on this one GPU, in one call: the
    exchange buffers are all local and a single launch runs every rank's
    second projection and exchange (their CTAs wait on one another, so they
    must share one launch).  Used to check the exchange on one GPU."""

    def __init__(self, d_model: int, d_ff: int, tp: int, act: str, max_tokens: int,
                 A_shards: Sequence[torch.Tensor], B_shards: Sequence[torch.Tensor], d_out: Optional[int] = None):
        from tensor_sharded_mlp_b200 import binding
        self.b = binding
        self.tp = tp
        self.A, self.B = list(A_shards), list(B_shards)
        self.mlp = binding.TpMlp(d_model, d_ff, tp, act, "bf16", max_tokens=max_tokens, d_out=d_out)
        nbytes = binding.tp_mlp_xgpu_comm_bytes(self.mlp.h)
        self.comm = [torch.zeros(nbytes, dtype=torch.uint8, device=self.mlp.device) for _ in range(tp)]
        self.ptrs = [c.data_ptr() for c in self.comm]

    def forward(self, x: torch.Tensor, stream=None) -> List[torch.Tensor]:
        outs = [torch.empty(x.shape[0], self.mlp.d_out, dtype=torch.bfloat16, device=x.device)
                for _ in range(self.tp)]
        self.b.tp_mlp_xgpu_forward(self.mlp.h, 0, x, self.A, self.B, self.ptrs, outs, stream)
        return outs

    def forward_sp(self, x: torch.Tensor, stream=None) -> List[torch.Tensor]:
        """Sequence-parallel form: rank r gets x's rows [r T/tp, (r+1) T/tp) and
        returns the same rows of the output."""
        rows = x.shape[0] // self.tp
        xs = [x[r * rows:(r + 1) * rows].contiguous() for r in range(self.tp)]
        outs = [torch.empty(rows, self.mlp.d_out, dtype=torch.bfloat16, device=x.device) for _ in range(self.tp)]
        self.b.tp_mlp_xgpu_sp_forward(self.mlp.h, 0, xs, self.A, self.B, self.ptrs, outs, stream)
        return outs
