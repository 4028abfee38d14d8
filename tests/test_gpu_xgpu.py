"""Tensor parallelism across GPUs with the one-shot all-reduce fused into the
second projection, checked on one GPU.

Every call here has one GPU, so every rank runs on it: a single launch holds
all ranks' second projections and exchanges (their CTAs wait on one another,
which is only sound inside one launch whose CTAs are all resident).  The
exchange buffers are then all local, but the code path -- per-rank partial
tiles stored into every rank's buffer, epoch flags, bounded waits, the sum in
rank order -- is the one a process per GPU runs.  Every rank's output must
match the oracle, all ranks must agree bit for bit, and consecutive calls
(epochs, alternating buffer halves) must stay correct.

The CUDA IPC helpers are checked with two processes on the same GPU that
share a buffer (no kernel waits on another).
"""
import os
import sys

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, dev
from tensor_sharded_mlp_b200 import inputs

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tensor_sharded_mlp_b200 import build
    build.build()


@pytest.mark.parametrize("act", ["swiglu", "tanh"])
@pytest.mark.parametrize("tp", [2, 4, 8])
@pytest.mark.parametrize("T", [1, 5, 16, 33, 128])
def test_emulated_ranks_match_the_oracle(act, tp, T):
    from tensor_sharded_mlp_b200 import binding as b, xgpu
    d, fs, dout = 256, 256, 1024
    f = tp * fs
    em = None
    for step in range(3):                       # calls 1, 2, 3: both buffer halves, then the first again
        p = inputs.generate(T, d, f, act, "bf16", seed=100 * step + 7 * tp + T, init="fan_in", d_out=dout)
        A, Bs = p.shards(tp)
        if em is None:
            Ad, Bd = [dev(a, "bf16") for a in A], [dev(x, "bf16") for x in Bs]
            em = xgpu.EmulatedRanks(d, f, tp, act, 128, Ad, Bd, d_out=dout)
            A0, B0 = A, Bs
        x = dev(p.x, "bf16")
        outs = em.forward(x)
        torch.cuda.synchronize()
        b.tp_mlp_get_device_status(em.mlp.h)    # no bounded wait ran out
        ref = oracle.tp_mlp_sharded(p.x, A0, B0, act)
        for r in range(tp):
            assert torch.equal(outs[r], outs[0]), f"rank {r} differs from rank 0"
        assert_close(outs[0], ref, "bf16", f"cross-GPU step, tp={tp}, T={T}, epoch {step + 1}")


@pytest.mark.parametrize("act", ["swiglu", "tanh"])
@pytest.mark.parametrize("tp,T", [(2, 2), (2, 34), (4, 16), (4, 128), (8, 8), (8, 64)])
def test_emulated_sequence_parallel_step(act, tp, T):
    """All-gather -> first projection, second projection -> reduce-scatter:
    rank r gets exactly rows [r T/tp, (r+1) T/tp) of the MLP's output.  The
    calls alternate with all-reduce calls on the same buffers."""
    from tensor_sharded_mlp_b200 import binding as b, xgpu
    d, fs, dout = 256, 256, 1024
    f = tp * fs
    em = None
    rows = T // tp
    for step in range(3):
        p = inputs.generate(T, d, f, act, "bf16", seed=300 + 11 * step + tp + T, init="fan_in", d_out=dout)
        A, Bs = p.shards(tp)
        if em is None:
            Ad, Bd = [dev(a, "bf16") for a in A], [dev(x, "bf16") for x in Bs]
            em = xgpu.EmulatedRanks(d, f, tp, act, 128, Ad, Bd, d_out=dout)
            A0, B0 = A, Bs
        x = dev(p.x, "bf16")
        outs = em.forward_sp(x)
        ar = em.forward(x)                      # an all-reduce call in between, same buffers
        torch.cuda.synchronize()
        b.tp_mlp_get_device_status(em.mlp.h)
        ref = oracle.tp_mlp_sharded(p.x, A0, B0, act)
        for r in range(tp):
            assert outs[r].shape == (rows, dout)
            assert_close(outs[r], ref[r * rows:(r + 1) * rows], "bf16", f"SP rank {r}, tp={tp}, T={T}, call {step}")
        assert_close(ar[0], ref, "bf16", f"all-reduce between SP calls, call {step}")
        # the same rows as the all-reduce form, bit for bit (same sums, same order)
        for r in range(tp):
            assert torch.equal(outs[r], ar[r][r * rows:(r + 1) * rows])


def test_emulated_step_agrees_with_the_single_gpu_forward_and_library_allreduce():
    from tensor_sharded_mlp_b200 import binding as b, xgpu
    d, f, dout, tp, T = 512, 4 * 512, 2048, 4, 32
    p = inputs.generate(T, d, f, "swiglu", "bf16", seed=3, init=0.02, d_out=dout)
    A, Bs = p.shards(tp)
    Ad, Bd = [dev(a, "bf16") for a in A], [dev(x, "bf16") for x in Bs]
    em = xgpu.EmulatedRanks(d, f, tp, "swiglu", T, Ad, Bd, d_out=dout)
    x = dev(p.x, "bf16")
    out = em.forward(x)[0]
    single = b.TpMlp(d, f, tp, "swiglu", "bf16", T, d_out=dout).forward(x, Ad, Bd)
    # the unfused step: each rank's fp32 partial, summed with a plain tensor sum (one process)
    parts = [xgpu.LibraryAllReduceMlp(d, f, tp, "swiglu", T, Ad[i], Bd[i], d_out=dout).one.partials(
        x, [Ad[i]], [Bd[i]])[0] for i in range(tp)]
    torch.cuda.synchronize()
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, "swiglu")
    assert_close(out, ref, "bf16", "fused exchange")
    assert_close(out, single.float().cpu().numpy(), "bf16", "fused exchange vs single-GPU forward")
    assert_close(torch.stack(parts).sum(0), ref, "bf16", "library partials summed")


def test_emulated_step_replays_in_a_cuda_graph():
    """The call count lives on the device, so one captured step replays
    correctly: each replay is the next epoch and uses the other buffer half."""
    from tensor_sharded_mlp_b200 import binding as b, xgpu
    d, fs, dout, tp, T = 256, 256, 1024, 4, 8
    f = tp * fs
    p = inputs.generate(T, d, f, "tanh", "bf16", seed=9, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    Ad, Bd = [dev(a, "bf16") for a in A], [dev(x, "bf16") for x in Bs]
    em = xgpu.EmulatedRanks(d, f, tp, "tanh", T, Ad, Bd, d_out=dout)
    x = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    outs = [torch.empty(T, dout, dtype=torch.bfloat16, device="cuda") for _ in range(tp)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        b.tp_mlp_xgpu_forward(em.mlp.h, 0, x, Ad, Bd, em.ptrs, outs)     # warm-up outside capture
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        b.tp_mlp_xgpu_forward(em.mlp.h, 0, x, Ad, Bd, em.ptrs, outs)
    for step in range(4):
        q = inputs.generate(T, d, f, "tanh", "bf16", seed=50 + step, init="fan_in", d_out=dout)
        x.copy_(dev(q.x, "bf16"))
        torch.cuda.synchronize()
        with torch.cuda.stream(s):
            g.replay()
        s.synchronize()
        b.tp_mlp_get_device_status(em.mlp.h)
        ref = oracle.tp_mlp_sharded(q.x, A, Bs, "tanh")
        for r in range(tp):
            assert_close(outs[r], ref, "bf16", f"graph replay {step}, rank {r}")
    del g


def test_errors_are_status_codes():
    from tensor_sharded_mlp_b200 import binding as b
    d, f, dout, tp = 128, 2 * 128, 256, 2
    m = b.TpMlp(d, f, tp, "tanh", "bf16", 8, d_out=dout)
    A = [torch.zeros(d, f // tp, dtype=torch.bfloat16, device="cuda") for _ in range(tp)]
    B = [torch.zeros(f // tp, dout, dtype=torch.bfloat16, device="cuda") for _ in range(tp)]
    comm = [torch.zeros(b.tp_mlp_xgpu_comm_bytes(m.h), dtype=torch.uint8, device="cuda") for _ in range(tp)]
    ptrs = [c.data_ptr() for c in comm]
    x = torch.zeros(4, d, dtype=torch.bfloat16, device="cuda")
    outs = [torch.zeros(4, dout, dtype=torch.bfloat16, device="cuda") for _ in range(tp)]
    with pytest.raises(b.TpMlpError):                  # ranks 1..2 of 2
        b.tp_mlp_xgpu_forward(m.h, 1, x, A, B, ptrs, outs)
    with pytest.raises(b.TpMlpError):                  # too many tokens for the handle
        b.tp_mlp_xgpu_forward(m.h, 0, torch.zeros(9, d, dtype=torch.bfloat16, device="cuda"), A, B, ptrs,
                              [torch.zeros(9, dout, dtype=torch.bfloat16, device="cuda")] * tp)
    # zero tokens: nothing runs
    b.tp_mlp_xgpu_forward(m.h, 0, torch.zeros(0, d, dtype=torch.bfloat16, device="cuda"), A, B, ptrs,
                          [torch.zeros(0, dout, dtype=torch.bfloat16, device="cuda")] * tp)
    torch.cuda.synchronize()
    assert all(int(c.count_nonzero()) == 0 for c in comm)


def _ipc_child(handle, offset, n, q):
    sys.path.insert(0, ROOT)
    import torch as t
    from cuda.bindings import runtime as rt
    from tensor_sharded_mlp_b200 import binding as b
    t.cuda.set_device(0)
    ptr = b.tp_mlp_ipc_open_handle(handle, offset)
    mine = t.empty(n, dtype=t.int32, device="cuda")      # a device-to-device copy into the child's own tensor
    err = rt.cudaMemcpy(mine.data_ptr(), ptr, n * 4, rt.cudaMemcpyKind.cudaMemcpyDeviceToDevice)[0]
    t.cuda.synchronize()
    vals = mine.cpu().tolist()
    b.tp_mlp_ipc_close_handle(ptr, offset)
    q.put((int(err), vals))


def test_ipc_handle_round_trip_between_two_processes():
    from tensor_sharded_mlp_b200 import binding as b
    import torch.multiprocessing as mp
    n = 1024
    base = torch.zeros(n + 4096, dtype=torch.int32, device="cuda")
    buf = base[4096:]                              # not at the start of its allocation: the offset matters
    buf.copy_(torch.arange(n, dtype=torch.int32, device="cuda") * 3 + 1)
    torch.cuda.synchronize()
    handle, offset = b.tp_mlp_ipc_get_handle(buf)
    assert len(handle) == 64 and offset >= 4096 * 4
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_ipc_child, args=(handle, offset, n, q))
    p.start()
    res, vals = q.get(timeout=120)
    p.join(timeout=120)
    assert res == 0
    assert vals == [3 * i + 1 for i in range(n)]
