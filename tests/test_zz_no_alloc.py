"""The decode entry point that allocates nothing (its scratch is a fixed
device array inside the library), checked against the regular packed forward.

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


@pytest.mark.parametrize("act,T", [("swiglu", 1), ("swiglu", 4), ("tanh", 3)])
def test_static_scratch_decode_matches_packed_forward(act, T):
    from tensor_sharded_mlp_b200 import binding as b
    d, f, dout, tp = 2048, 4096, 1024, 4
    p = inputs.generate(T, d, f, act, "bf16", seed=40 + T, init=0.02, d_out=dout)
    A, Bs = p.shards(tp)
    m = b.TpMlp(d, f, tp, act, "bf16", max_tokens=4, d_out=dout)
    m.set_plan("gemv")
    packed = m.pack([dev(a, "bf16") for a in A], [dev(x, "bf16") for x in Bs])
    x = dev(p.x, "bf16")
    want = m.forward_packed(x, packed)
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, act)
    for _ in range(2):   # two calls in a row share (and reuse) the scratch array
        out = torch.full((T, dout), float("nan"), dtype=torch.bfloat16, device="cuda")
        b.tp_mlp_decode_forward_static(d, f, dout, tp, act, x, packed, out)
        torch.cuda.synchronize()
        assert_close(out, want.float().cpu().numpy(), "bf16", "static vs packed forward")
        assert_close(out, ref, "bf16", "static vs oracle")


def test_static_scratch_rejects_shapes_beyond_its_size():
    from tensor_sharded_mlp_b200 import binding as b
    d, f = 64, 1 << 22          # H alone would need 4 tokens x 4M x 2 bytes = 32 MiB
    x = torch.zeros(4, d, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(4, d, dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(b.TpMlpError) as ei:
        b.tp_mlp_decode_forward_static(d, f, d, 1, "tanh", x, packed, out)
    assert ei.value.name == "ERR_WORKSPACE"
