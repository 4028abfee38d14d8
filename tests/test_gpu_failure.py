"""Failure detection on the GPU without a GPU fault.

A kernel waits, through the bounded mbarrier wait every pipelined kernel here
uses, on a barrier nothing completes; the wait runs out after a short limit,
the kernel records the timeout and returns.  The host reads the status as
TP_MLP_ERR_TIMEOUT, and the context keeps working.
"""
import pytest
import torch

import oracle
from helpers import assert_close, dev
from tensor_sharded_mlp_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tensor_sharded_mlp_b200 import build
    build.build()


def test_bounded_wait_times_out_and_reports_status():
    from tensor_sharded_mlp_b200 import binding as b
    p = inputs.generate(2, 256, 512, "swiglu", "bf16", seed=21)
    A, Bs = p.shards(2)
    m = b.TpMlp(256, 512, 2, "swiglu", "bf16", max_tokens=2)
    b.tp_mlp_get_device_status(m.h)                 # clean to start with
    b.tp_mlp_selftest_bounded_wait(m.h, 2000)       # 2 ms limit on a barrier nobody arrives at
    with pytest.raises(b.TpMlpError) as ei:
        b.tp_mlp_get_device_status(m.h)
    assert ei.value.name == "ERR_TIMEOUT"
    b.tp_mlp_get_device_status(m.h)                 # reading cleared it
    # the context is still healthy: a normal forward runs and is correct
    packed = m.pack([dev(a, "bf16") for a in A], [dev(x, "bf16") for x in Bs])
    out = m.forward_packed(dev(p.x, "bf16"), packed)
    torch.cuda.synchronize()
    assert_close(out, oracle.tp_mlp_sharded(p.x, A, Bs, "swiglu"), "bf16", "after the timeout")
    b.tp_mlp_get_device_status(m.h)


def test_selftest_argument_checks():
    from tensor_sharded_mlp_b200 import binding as b
    m = b.TpMlp(64, 128, 2, "tanh", "bf16", max_tokens=1)
    for bad in (0, 100001):
        with pytest.raises(b.TpMlpError):
            b.tp_mlp_selftest_bounded_wait(m.h, bad)


@pytest.mark.parametrize("plan,T,splitk", [("gemv", 1, "auto"), ("gemv", 3, "auto"), ("tc_skinny", 16, "in_kernel")])
def test_timeout_report_resets_split_tile_counters(plan, T, splitk):
    """After a bounded wait runs out, CTAs that left early can leave split-tile
    counters part-way.  Injected on the host: the caller-owned workspace's
    counter region (its first tp_mlp_workspace_bytes(h, 0) bytes, status word
    included) is filled with garbage.  The status call must report the timeout
    and restore the counters, so the next forward matches the oracle."""
    from tensor_sharded_mlp_b200 import binding as b
    d, f, tp = 1024, 4096, 4
    p = inputs.generate(T, d, f, "swiglu", "bf16", seed=60 + T, init=0.02)
    A, Bs = p.shards(tp)
    m = b.TpMlp(d, f, tp, "swiglu", "bf16", max_tokens=T)
    m.set_plan(plan)
    m.set_splitk(splitk)
    packed = m.pack([dev(a, "bf16") for a in A], [dev(x, "bf16") for x in Bs])
    x = dev(p.x, "bf16")
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, "swiglu")
    assert_close(m.forward_packed(x, packed), ref, "bf16", "before the injection")
    n0 = b.tp_mlp_workspace_bytes(m.h, 0)
    assert 0 < n0 <= m.workspace.numel()
    torch.cuda.synchronize()
    m.workspace[:n0].fill_(0xFF)
    with pytest.raises(b.TpMlpError) as ei:
        b.tp_mlp_get_device_status(m.h)
    assert ei.value.name == "ERR_TIMEOUT"
    assert int(m.workspace[:n0].count_nonzero()) == 0
    for _ in range(2):
        out = m.forward_packed(x, packed)
        torch.cuda.synchronize()
        assert_close(out, ref, "bf16", "after the counters were reset")
        # the kernels leave every counter at zero again
        assert int(m.workspace[:n0].count_nonzero()) == 0
    b.tp_mlp_get_device_status(m.h)
