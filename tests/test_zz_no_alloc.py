"""The decode entry point that allocates nothing (its scratch is a fixed
device array inside the library), checked against the regular packed forward.

Some callers cannot allocate device memory -- code inside host callbacks or
allocator hooks, plugins whose host owns every allocation -- so they cannot
hand the library a workspace; this entry point serves them.

Collected last on purpose.  It must pass alone in a fresh process and after
the rest of the suite.
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


def _check_against_packed(d, f, dout, tp, act, T, seed, stream=None, calls=2):
    from tensor_sharded_mlp_b200 import binding as b
    p = inputs.generate(T, d, f, act, "bf16", seed=seed, init=0.02, d_out=dout)
    A, Bs = p.shards(tp)
    m = b.TpMlp(d, f, tp, act, "bf16", max_tokens=4, d_out=dout)
    m.set_plan("gemv")
    packed = m.pack([dev(a, "bf16") for a in A], [dev(x, "bf16") for x in Bs])
    x = dev(p.x, "bf16")
    want = m.forward_packed(x, packed)
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, act)
    torch.cuda.synchronize()
    for _ in range(calls):   # calls in a row share (and reuse) the scratch array
        out = torch.full((T, dout), float("nan"), dtype=torch.bfloat16, device="cuda")
        if stream is None:
            b.tp_mlp_decode_forward_static(d, f, dout, tp, act, x, packed, out)
            torch.cuda.synchronize()
        else:
            stream.wait_stream(torch.cuda.current_stream())
            b.tp_mlp_decode_forward_static(d, f, dout, tp, act, x, packed, out, stream=stream)
            stream.synchronize()
        assert_close(out, want.float().cpu().numpy(), "bf16", "static vs packed forward")
        assert_close(out, ref, "bf16", "static vs oracle")
    b.tp_mlp_decode_static_status()   # no bounded wait ran out


@pytest.mark.parametrize("act,T", [("swiglu", 1), ("swiglu", 4), ("tanh", 3)])
def test_static_scratch_decode_matches_packed_forward(act, T):
    _check_against_packed(2048, 4096, 1024, 4, act, T, seed=40 + T)


def test_static_scratch_on_a_side_stream():
    _check_against_packed(2048, 4096, 2048, 8, "swiglu", 2, seed=47, stream=torch.cuda.Stream())


def _static_status_name(d, f, dout, tp, T):
    """Which check a call of this shape stops at, through the C entry point with
    x in host memory: ERR_WORKSPACE if its scratch does not fit the array,
    otherwise ERR_INVALID_ARG from the check that x is device memory, which
    comes next.  Either way nothing launches."""
    import ctypes

    import numpy as np

    from tensor_sharded_mlp_b200 import binding as b
    host = np.zeros(T * d + 64, dtype=np.uint16)                   # pageable host memory
    off = (-host.ctypes.data % 16) // 2                             # 16-byte aligned start
    x_host = ctypes.c_void_p(host.ctypes.data + 2 * off)
    out = torch.zeros(T, dout, dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros(16, dtype=torch.uint8, device="cuda")
    st = b._stream(None)
    code = b._lib.tp_mlp_decode_forward_static(d, f, dout, tp, b.ACT["tanh"], x_host, T,
                                               ctypes.c_void_p(packed.data_ptr()), ctypes.c_void_p(out.data_ptr()), st)
    return b.STATUS.get(code, str(code))


def test_static_scratch_largest_shape_that_fits():
    """Search d_ff (multiples of 8, 4 tokens) for the largest shape whose
    scratch fits the array, run that shape for real, and check that the next
    larger one is rejected."""
    d, dout, tp, T = 256, 256, 8, 4
    lo, hi = 1, 1 << 20                     # d_ff = 8 lo fits; 8 hi (8M features) cannot
    assert _static_status_name(d, 8 * lo, dout, tp, T) == "ERR_INVALID_ARG"
    assert _static_status_name(d, 8 * hi, dout, tp, T) == "ERR_WORKSPACE"
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if _static_status_name(d, 8 * mid, dout, tp, T) == "ERR_WORKSPACE":
            hi = mid
        else:
            lo = mid
    f = 8 * lo
    assert f >= 65536, f"only d_ff={f} fits at 4 tokens"
    assert _static_status_name(d, f + 8, dout, tp, T) == "ERR_WORKSPACE"
    _check_against_packed(d, f, dout, tp, "tanh", T, seed=48, calls=2)


def test_static_scratch_rejects_shapes_beyond_its_size():
    assert _static_status_name(64, 1 << 22, 64, 1, 4) == "ERR_WORKSPACE"   # H alone: 32 MiB
