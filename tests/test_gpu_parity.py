"""GPU parity: the CUDA library against the oracle on the same seeded inputs.

Every test calls the library through its C ABI (via the thin binding) and
compares element by element with the fp64 oracle, under the rule in
tests/helpers.py (1e-5 for fp32, 2e-2 for bf16, relative to max |ref|), or
bit-exactly where the arithmetic is exact (integer cases, the packer).
"""
import numpy as np
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


def B():
    from tensor_sharded_mlp_b200 import binding
    return binding


def _upload(p, tp, dtype):
    A, Bs = p.shards(tp)
    return [dev(a, dtype) for a in A], [dev(b, dtype) for b in Bs], A, Bs


def _mlp(p, tp, dtype, max_tokens=None):
    return B().TpMlp(p.d_in, p.d_ff, tp, p.act, dtype, max_tokens or max(1, p.tokens), d_out=p.d_out)


# --- the small fp32 workload ---------------------------------------------------

def test_tiny_config_all_entry_points():
    c = inputs.CONFIGS["tiny"]
    p = inputs.generate_config("tiny")
    tp = c["tp"]
    Ad, Bd, A, Bs = _upload(p, tp, "f32")
    ref, parts = oracle.tp_mlp_sharded(p.x, A, Bs, "tanh", return_partials=True)
    m = _mlp(p, tp, "f32")
    x = dev(p.x, "f32")
    assert_close(m.forward(x, Ad, Bd), ref, "f32", "forward")
    assert m.last_plan == "simt"
    gp = m.partials(x, Ad, Bd)
    for i in range(tp):
        assert_close(gp[i], parts[i], "f32", f"partial {i}")
    assert_close(gp.sum(0), ref, "f32", "sum of partials")
    packed = m.pack(Ad, Bd)
    assert_close(m.forward_packed(x, packed), ref, "f32", "forward_packed")


# --- exact cases -----------------------------------------------------------------

@pytest.mark.parametrize("act", ["identity", "swiglu"])
@pytest.mark.parametrize("tp", [1, 2, 4, 8])
def test_integer_inputs_fp32_bit_exact(act, tp):
    """Small integers: every sum is exact in fp32, so GPU == oracle bit for bit,
    and the partials sum exactly.  SwiGLU uses gate = 0 (SiLU(0) = 0 exactly)."""
    p = inputs.integer_inputs(5, 40, 8 * tp * 3, 24, act, seed=tp)
    if act == "swiglu":
        p.gate[:] = 0.0
    Ad, Bd, A, Bs = _upload(p, tp, "f32")
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, act)
    m = _mlp(p, tp, "f32")
    x = dev(p.x, "f32")
    assert np.array_equal(m.forward(x, Ad, Bd).cpu().numpy().astype(np.float64), ref)
    assert np.array_equal(m.partials(x, Ad, Bd).sum(0).cpu().numpy().astype(np.float64), ref)
    packed = m.pack(Ad, Bd)
    assert np.array_equal(m.forward_packed(x, packed).cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("plan", ["simt", "gemv", "tc_pair", "tc_pair2"])
@pytest.mark.parametrize("T", [1, 3, 4])
def test_integer_inputs_bf16_exact_rounding(plan, T):
    """bf16 with |H| <= 64 (exact in bf16) and fp32 sums that stay exact: the
    only rounding is the final one, so GPU == round_to_bf16(oracle) exactly."""
    p = inputs.integer_inputs(T, 16, 64, 40, "identity", seed=T, lo=-2, hi=2)
    Ad, Bd, A, Bs = _upload(p, 4, "bf16")
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, "identity")
    want = inputs.round_to_bf16(ref.astype(np.float32))
    m = _mlp(p, 4, "bf16")
    m.set_plan(plan)
    packed = m.pack(Ad, Bd)
    got = m.forward_packed(dev(p.x, "bf16"), packed).float().cpu().numpy()
    assert m.last_plan == plan
    assert np.array_equal(got, want)


# --- the shard-layout packer -----------------------------------------------------------

def _blocked(mat, esize):
    """A part (rows x K) in the tile-blocked order the header documents:
    256-row tiles, 64-wide k-blocks, each 256 x 64 block contiguous."""
    R, K = mat.shape
    tiles, kbs = -(-R // 256), -(-K // 64)
    pad = np.zeros((tiles * 256, kbs * 64), np.float32)
    pad[:R, :K] = mat
    blk = np.ascontiguousarray(pad.reshape(tiles, 256, kbs, 64).transpose(0, 2, 1, 3))
    raw = blk.view(np.uint32) if esize == 4 else (blk.view(np.uint32) >> 16).astype(np.uint16)
    return np.frombuffer(raw.tobytes(), np.uint8)


def _expected_packed(p, tp, esize):
    """The packed buffer as the header documents it, built on the host."""
    def a256(v):
        return (v + 255) // 256 * 256
    f, d = p.d_ff, p.d_in
    if p.act == "swiglu":
        nb = -(-f // 128)
        part1 = np.zeros((256 * nb, d), np.float32)
        for n in range(f):
            b, r = divmod(n, 128)
            part1[256 * b + r] = p.gate[:, n]
            part1[256 * b + 128 + r] = p.up[:, n]
    else:
        part1 = p.a.T
    part2 = p.b.T          # row c = column c of B over all ranks' rows in rank order
    b1, b2 = _blocked(part1, esize), _blocked(part2, esize)
    off = a256(b1.size)
    buf = np.zeros(off + a256(b2.size), np.uint8)
    buf[:b1.size] = b1
    buf[off:off + b2.size] = b2
    return buf, off, b1.size, b2.size


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("act", ["tanh", "swiglu", "identity"])
@pytest.mark.parametrize("tp", [1, 2, 4, 8])
def test_pack_layout_and_roundtrip_bit_exact(dtype, act, tp):
    p = inputs.generate(3, 40, 400, act, dtype, seed=tp + 10, d_out=24)   # f = 400: ragged 128-blocks
    Ad, Bd, A, Bs = _upload(p, tp, dtype)
    m = _mlp(p, tp, dtype)
    packed = m.pack(Ad, Bd)
    want, off, n1, n2 = _expected_packed(p, tp, 4 if dtype == "f32" else 2)
    got = packed.cpu().numpy()
    assert got.size == want.size
    assert np.array_equal(got[:n1], want[:n1])
    assert np.array_equal(got[off:off + n2], want[off:off + n2])
    A2, B2 = m.unpack(packed)
    for a, a2 in zip(Ad, A2):
        assert torch.equal(a.view(torch.int16 if dtype == "bf16" else torch.int32),
                           a2.view(torch.int16 if dtype == "bf16" else torch.int32))
    for b, b2 in zip(Bd, B2):
        assert torch.equal(b.view(torch.int16 if dtype == "bf16" else torch.int32),
                           b2.view(torch.int16 if dtype == "bf16" else torch.int32))


# --- bf16 parity across paths, tiles and ragged tails --------------------------------

GEMV_SHAPES = [  # (d_in, d_ff, d_out, tp)
    (1024, 2048, 1024, 4),
    (520, 400, 264, 4),      # K not a multiple of 256, ragged 128-blocks
    (8192, 1024, 256, 2),    # long K: split-K in the first projection at T >= 3
    (256, 4096, 128, 8),     # few output rows: split-K in the second projection
    (136, 38400, 200, 4),    # K of 3 blocks, the last ragged: shares longer than K, staged X windows wrap
]


@pytest.mark.parametrize("act", ["tanh", "swiglu", "identity"])
@pytest.mark.parametrize("T", [1, 2, 3, 4])
@pytest.mark.parametrize("shape", GEMV_SHAPES)
def test_gemv_decode_parity(act, T, shape):
    d, f, dout, tp = shape
    p = inputs.generate(T, d, f, act, "bf16", seed=T + d, init="fan_in", d_out=dout)
    Ad, Bd, A, Bs = _upload(p, tp, "bf16")
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, act)
    m = _mlp(p, tp, "bf16", max_tokens=4)
    packed = m.pack(Ad, Bd)
    x = dev(p.x, "bf16")
    m.set_plan("gemv")
    got = m.forward_packed(x, packed)
    assert m.last_plan == "gemv" and m.last_launches == 2
    assert_close(got, ref, "bf16", "gemv")
    again = m.forward_packed(x, packed)           # split-K counters were reset
    assert torch.equal(got, again)


@pytest.mark.slow
def test_gemv_window_too_large_for_shared_memory():
    """4 tokens, K = 12160 and 148 tiles of the first projection: a CTA's share
    is a whole tile's K (190 blocks), whose X (4 x 190 x 128 B) no longer fits
    beside the weight ring, so that projection reads X from L2 instead."""
    T, d, f, dout, tp = 4, 12160, 37888, 256, 4
    p = inputs.generate(T, d, f, "tanh", "bf16", seed=11, init="fan_in", d_out=dout)
    Ad, Bd, A, Bs = _upload(p, tp, "bf16")
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, "tanh")
    del A, Bs
    m = _mlp(p, tp, "bf16", max_tokens=T)
    m.set_plan("gemv")
    got = m.forward_packed(dev(p.x, "bf16"), m.pack(Ad, Bd))
    assert m.last_plan == "gemv"
    assert_close(got, ref, "bf16", "gemv, X read from L2")


@pytest.mark.parametrize("act", ["tanh", "swiglu"])
@pytest.mark.parametrize("T", [1, 17, 40])
def test_simt_bf16_parity(act, T):
    p = inputs.generate(T, 200, 8 * 33, act, "bf16", seed=T, init="fan_in", d_out=72)
    Ad, Bd, A, Bs = _upload(p, 4, "bf16")
    ref, parts = oracle.tp_mlp_sharded(p.x, A, Bs, act, return_partials=True)
    m = _mlp(p, 4, "bf16")
    x = dev(p.x, "bf16")
    assert_close(m.forward(x, Ad, Bd), ref, "bf16", "shard form")
    gp = m.partials(x, Ad, Bd)
    assert_close(gp.sum(0), ref, "bf16", "partials")
    m.set_plan("simt")
    assert_close(m.forward_packed(x, m.pack(Ad, Bd)), ref, "bf16", "packed simt")


def test_auto_plan_choice():
    p = inputs.generate(4, 256, 512, "swiglu", "bf16", seed=1)
    Ad, Bd, _, _ = _upload(p, 2, "bf16")
    m = _mlp(p, 2, "bf16", max_tokens=64)
    packed = m.pack(Ad, Bd)
    m.forward_packed(dev(p.x[:1], "bf16"), packed)
    assert m.last_plan == "gemv"
    m.forward_packed(dev(p.x[:3], "bf16"), packed)
    assert m.last_plan == "tc_fused"


# --- the named workloads at full size ---------------------------------------------------

@pytest.mark.slow
@pytest.mark.parametrize("name", ["decode_bs1", "decode_bs32"])
def test_decode_configs_full_size(name):
    c = inputs.CONFIGS[name]
    p = inputs.generate_config(name)
    Ad, Bd, A, Bs = _upload(p, c["tp"], "bf16")
    ref, parts = oracle.tp_mlp_sharded(p.x, A, Bs, "swiglu", return_partials=True)
    m = _mlp(p, c["tp"], "bf16", max_tokens=32)
    x = dev(p.x, "bf16")
    packed = m.pack(Ad, Bd)
    del A, Bs
    assert_close(m.forward_packed(x, packed), ref, "bf16", f"{name} packed/{m.last_plan}")
    if c["tokens"] > 1:   # the two-kernel skinny tiling (auto takes the fused one)
        m.set_plan("tc_skinny")
        assert_close(m.forward_packed(x, packed), ref, "bf16", f"{name} packed/tc_skinny")
        m.set_plan("auto")
    out = m.forward(x, Ad, Bd)
    assert_close(out, ref, "bf16", f"{name} shard form")
    # the per-rank partials (tensor cores, each rank's K loop apart) and their sum
    gp = m.partials(x, Ad, Bd)
    assert m.last_plan == "tc_skinny"
    for i in range(c["tp"]):
        assert_close(gp[i], parts[i], "bf16", f"{name} partial {i}")
    assert_close(gp.sum(0), ref, "bf16", f"{name} sum of partials")
    assert_close(out, gp.sum(0).cpu().numpy(), "bf16", f"{name} forward vs sum of partials")


@pytest.mark.slow
@pytest.mark.parametrize("T", [1, 16, 128, 1024, 4096])
def test_sweep_config(T):
    c = inputs.CONFIGS["sweep"]
    p = inputs.generate_config("sweep", tokens=T)
    rows = p.sample_rows(16)
    ref = None
    for tp in c["tp"]:
        Ad, Bd, A, Bs = _upload(p, tp, "bf16")
        if ref is None:
            ref = oracle.tp_mlp_sharded(p.x[rows], A, Bs, "tanh")
        m = _mlp(p, tp, "bf16", max_tokens=T)
        x = dev(p.x, "bf16")
        packed = m.pack(Ad, Bd)
        out = m.forward_packed(x, packed)
        assert_close(out[torch.from_numpy(rows).cuda()], ref, "bf16", f"sweep T={T} tp={tp}")
        if 1 < T <= 128:   # the two-kernel skinny tiling (auto takes the fused one)
            m.set_plan("tc_skinny")
            out = m.forward_packed(x, packed)
            assert_close(out[torch.from_numpy(rows).cuda()], ref, "bf16", f"sweep T={T} tp={tp} skinny")
            m.set_plan("auto")
        out = m.forward(x, Ad, Bd)          # the shard form (its own tiling and grid)
        assert_close(out[torch.from_numpy(rows).cuda()], ref, "bf16", f"sweep T={T} tp={tp} shard form")
        del Ad, Bd, m


@pytest.mark.slow
def test_prefill_config_sampled_rows():
    c = inputs.CONFIGS["prefill"]
    p = inputs.generate_config("prefill")
    rows = p.sample_rows(c["sample_rows"])
    ref = None
    for tp in c["tp"]:
        Ad, Bd, A, Bs = _upload(p, tp, "bf16")
        if ref is None:
            ref = oracle.tp_mlp_sharded(p.x[rows], A, Bs, "swiglu")
        m = _mlp(p, tp, "bf16", max_tokens=p.tokens)
        x = dev(p.x, "bf16")
        out = m.forward_packed(x, m.pack(Ad, Bd))
        r = torch.from_numpy(rows).cuda()
        assert_close(out[r], ref, "bf16", f"prefill tp={tp}/{m.last_plan}")
        if tp == 8:
            # per-rank partials of all 8192 rows (fp32, 2 GiB), checked on the sample
            _, parts = oracle.tp_mlp_sharded(p.x[rows], A, Bs, "swiglu", return_partials=True)
            gp = m.partials(x, Ad, Bd)
            assert m.last_plan == "tc_wide256"
            for i in range(tp):
                assert_close(gp[i][r], parts[i], "bf16", f"prefill partial {i}")
            assert_close(gp.sum(0)[r], ref, "bf16", "prefill sum of partials")
            del gp
        del Ad, Bd, m, out
        torch.cuda.empty_cache()


# --- behaviour ------------------------------------------------------------------------------

def test_errors_are_status_codes_not_launches():
    b = B()
    p = inputs.generate(2, 64, 128, "tanh", "bf16", seed=0)
    Ad, Bd, _, _ = _upload(p, 2, "bf16")
    m = _mlp(p, 2, "bf16", max_tokens=2)
    x = dev(p.x, "bf16")
    out = torch.empty(2, 64, dtype=torch.bfloat16, device="cuda")
    # misaligned x (one element in)
    xm = torch.empty(2 * 64 + 1, dtype=torch.bfloat16, device="cuda")[1:].view(2, 64)
    with pytest.raises(b.TpMlpError) as ei:
        b.tp_mlp_forward(m.h, xm, Ad, Bd, 2, "tanh", out)
    assert ei.value.name == "ERR_ALIGNMENT"
    # host memory where device memory is required
    with pytest.raises(b.TpMlpError) as ei:
        b.tp_mlp_forward(m.h, x.cpu(), Ad, Bd, 2, "tanh", out)
    assert ei.value.name == "ERR_INVALID_ARG"
    # more tokens than the handle was made for
    with pytest.raises(b.TpMlpError) as ei:
        b.tp_mlp_forward(m.h, dev(np.zeros((3, 64), np.float32), "bf16"), Ad, Bd, 2, "tanh",
                         torch.empty(3, 64, dtype=torch.bfloat16, device="cuda"))
    assert ei.value.name == "ERR_SHAPE"
    # workspace smaller than this call needs
    h = b.tp_mlp_create(64, 128, 64, 2, "tanh", "bf16", 2)
    small = torch.empty(b.tp_mlp_workspace_bytes(h, 1), dtype=torch.uint8, device="cuda")
    b.tp_mlp_set_workspace(h, small)
    with pytest.raises(b.TpMlpError) as ei:
        b.tp_mlp_forward(h, x, Ad, Bd, 2, "tanh", out)
    assert ei.value.name == "ERR_WORKSPACE"
    b.tp_mlp_destroy(h)
    torch.cuda.synchronize()
    # the context is still healthy
    assert torch.isfinite(m.forward(x, Ad, Bd).float()).all()


def test_zero_tokens_is_a_no_op():
    p = inputs.generate(1, 64, 128, "tanh", "bf16", seed=0)
    Ad, Bd, _, _ = _upload(p, 2, "bf16")
    m = _mlp(p, 2, "bf16")
    out = m.forward(torch.empty(0, 64, dtype=torch.bfloat16, device="cuda"), Ad, Bd)
    assert out.shape == (0, 64) and m.last_launches == 0


def test_cuda_graph_replay_matches_eager():
    p = inputs.generate(2, 512, 1024, "swiglu", "bf16", seed=5)
    Ad, Bd, A, Bs = _upload(p, 4, "bf16")
    m = _mlp(p, 4, "bf16", max_tokens=2)
    packed = m.pack(Ad, Bd)
    x = dev(p.x, "bf16")
    eager = m.forward_packed(x, packed)
    out = torch.empty_like(eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        m.forward_packed(x, packed, out=out)      # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        m.forward_packed(x, packed, out=out)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)


def test_profile_events_bracket_the_kernels():
    b = B()
    p = inputs.generate(1, 1024, 4096, "swiglu", "bf16", seed=6)
    Ad, Bd, _, _ = _upload(p, 4, "bf16")
    m = _mlp(p, 4, "bf16", max_tokens=1)
    packed = m.pack(Ad, Bd)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for e in ev:
        e.record()
    b.tp_mlp_set_profile_events(m.h, ev)
    m.forward_packed(dev(p.x, "bf16"), packed)
    b.tp_mlp_set_profile_events(m.h, None)
    torch.cuda.synchronize()
    assert ev[0].elapsed_time(ev[1]) > 0 and ev[1].elapsed_time(ev[2]) > 0


def test_graph_step_replays_copies_and_forward():
    b = B()
    p = inputs.generate(2, 512, 1024, "swiglu", "bf16", seed=8)
    A, Bs = p.shards(4)
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, "swiglu")
    m = b.TpMlp(512, 1024, 4, "swiglu", "bf16", max_tokens=2)
    packed = m.pack([dev(a, "bf16") for a in A], [dev(x, "bf16") for x in Bs])
    step = b.GraphStep(m, packed, 2)
    x = torch.from_numpy(p.x).to(torch.bfloat16)
    first = step(x).clone()
    assert_close(first, ref, "bf16", "graph step")
    assert torch.equal(first, m.forward_packed(x.cuda(), packed).cpu())
    # every call must wait for its own result: a new input must show up at once
    for sign in (-1.0, 1.0, -1.0):
        step.out_host.fill_(float("nan"))
        got = step(sign * x)
        assert torch.isfinite(got.float()).all()
        want = m.forward_packed((sign * x).cuda(), packed).cpu()
        assert torch.equal(got, want)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_page_worked_example_shapes(dtype):
    """"大模型推理系统揭秘（07）" §1.2.3: X in R^{Bx8}, W1 8x8 split by columns into
    four 8x2 blocks, W2 8x4 split by rows into four 2x4 blocks (d_out = 4 != d_in)."""
    for act in ("identity", "tanh", "swiglu"):
        p = inputs.generate(3, 8, 8, act, dtype, seed=11, init="fan_in", d_out=4)
        A, Bs = p.shards(4)
        ref = oracle.tp_mlp_sharded(p.x, A, Bs, act)
        m = B().TpMlp(8, 8, 4, act, dtype, max_tokens=3, d_out=4)
        Ad, Bd = [dev(a, dtype) for a in A], [dev(b, dtype) for b in Bs]
        x = dev(p.x, dtype)
        assert_close(m.forward(x, Ad, Bd), ref, dtype, f"{act} shard form")
        parts = m.partials(x, Ad, Bd)
        assert_close(parts.sum(0), ref, dtype, f"{act} partials")
        packed = m.pack(Ad, Bd)
        for T in (1, 3):
            r = oracle.tp_mlp_sharded(p.x[:T], A, Bs, act)
            assert_close(m.forward_packed(x[:T], packed), r, dtype, f"{act} packed T={T} ({m.last_plan})")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_one_feature_per_rank(dtype):
    """Degenerate split: d_ff == tp, so every rank holds a single feature."""
    p = inputs.generate(5, 16, 8, "tanh", dtype, seed=12, init="fan_in", d_out=24)
    A, Bs = p.shards(8)
    assert all(a.shape == (16, 1) for a in A)
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, "tanh")
    m = B().TpMlp(16, 8, 8, "tanh", dtype, max_tokens=5, d_out=24)
    Ad, Bd = [dev(a, dtype) for a in A], [dev(b, dtype) for b in Bs]
    assert_close(m.forward(dev(p.x, dtype), Ad, Bd), ref, dtype, "shard form")
    assert_close(m.forward_packed(dev(p.x, dtype), m.pack(Ad, Bd)), ref, dtype, f"packed ({m.last_plan})")
