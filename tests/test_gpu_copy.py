"""GPU checks of tp_mlp_copy_async, the host<->device copy of a step's input and
output: bytes arrive unchanged in every direction and at every size (kernel
copies up to 1 MiB with a ragged tail, copy-engine copies above), a captured
step (GraphStep) gives what the forward gives, and bad arguments are rejected
on the host before anything is launched.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tensor_sharded_mlp_b200 import build
    build.build()


def B():
    from tensor_sharded_mlp_b200 import binding
    return binding


SIZES = [16, 48, 1000, 16384, 16384 + 5, 524288, 1 << 20, (1 << 20) + 16, 3 * (1 << 20) + 7]


@pytest.mark.parametrize("nbytes", SIZES)
def test_copy_every_direction_is_exact(nbytes):
    g = torch.Generator().manual_seed(nbytes)
    src = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, generator=g).pin_memory()
    dev = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    dev2 = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    back = torch.zeros(nbytes, dtype=torch.uint8).pin_memory()
    s = torch.cuda.Stream()
    B().tp_mlp_copy_async(dev, src, stream=s)        # host -> device
    B().tp_mlp_copy_async(dev2, dev, stream=s)       # device -> device
    B().tp_mlp_copy_async(back, dev2, stream=s)      # device -> host
    s.synchronize()
    assert torch.equal(dev.cpu(), src)
    assert torch.equal(back, src)


def test_copies_in_a_graph_replay_with_new_host_data():
    n = 4096
    src = torch.zeros(n, dtype=torch.uint8).pin_memory()
    back = torch.zeros(n, dtype=torch.uint8).pin_memory()
    dev = torch.zeros(n, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        B().tp_mlp_copy_async(dev, src)
        B().tp_mlp_copy_async(back, dev)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        B().tp_mlp_copy_async(dev, src)
        B().tp_mlp_copy_async(back, dev)
    for seed in range(3):
        src.copy_(torch.randint(0, 256, (n,), dtype=torch.uint8, generator=torch.Generator().manual_seed(seed)))
        with torch.cuda.stream(s):
            g.replay()
        s.synchronize()
        assert torch.equal(back, src)


@pytest.mark.parametrize("act,tokens,d", [("swiglu", 1, 256), ("swiglu", 3, 256), ("tanh", 16, 256),
                                          ("tanh", 160, 4096)])   # x and out of 1.25 MiB: copy-engine copies
def test_graph_step_matches_the_forward(act, tokens, d):
    f, tp = 1024, 4
    m = B().TpMlp(d, f, tp, act, "bf16", max_tokens=max(16, tokens))
    fs = f // tp
    wa = 2 * fs if act == "swiglu" else fs
    g = torch.Generator().manual_seed(tokens)
    A = [(torch.randn(d, wa, generator=g) * 0.05).to(torch.bfloat16).cuda() for _ in range(tp)]
    Bs = [(torch.randn(fs, d, generator=g) * 0.05).to(torch.bfloat16).cuda() for _ in range(tp)]
    packed = m.pack(A, Bs)
    x = torch.randn(tokens, d, generator=g).to(torch.bfloat16)
    ref = m.forward_packed(x.cuda(), packed)
    torch.cuda.synchronize()
    step = B().GraphStep(m, packed, tokens)
    for _ in range(2):
        out = step(x)
        assert torch.equal(out, ref.cpu())


def test_copy_rejects_bad_arguments_before_launch():
    L = B()._lib
    vp = ctypes.c_void_p
    host = torch.zeros(4096, dtype=torch.uint8).pin_memory()          # one 4 KB pinned block
    dev = torch.zeros(4096, dtype=torch.uint8, device="cuda")         # inside a 2 MB allocator segment
    big_host = torch.zeros(4 << 20, dtype=torch.uint8).pin_memory()
    big_dev = torch.zeros(4 << 20, dtype=torch.uint8, device="cuda")
    assert L.tp_mlp_copy_async(vp(dev.data_ptr()), vp(host.data_ptr()), 4096, None) == 0
    torch.cuda.synchronize()
    # past the end of the pinned block
    assert L.tp_mlp_copy_async(vp(big_dev.data_ptr()), vp(host.data_ptr()), 4 << 20, None) == 2
    # past the end of the device segment
    assert L.tp_mlp_copy_async(vp(big_host.data_ptr()), vp(dev.data_ptr()), (2 << 20) + 16, None) == 2
    # misaligned, overlapping
    assert L.tp_mlp_copy_async(vp(dev.data_ptr() + 8), vp(host.data_ptr()), 64, None) == 3
    assert L.tp_mlp_copy_async(vp(big_dev.data_ptr() + 16), vp(big_dev.data_ptr()), 64, None) == 1
    # the binding refuses pageable host tensors before calling the library
    with pytest.raises(ValueError):
        B().tp_mlp_copy_async(dev, torch.zeros(4096, dtype=torch.uint8))
    with pytest.raises(ValueError):
        B().tp_mlp_copy_async(dev, host[:100])
