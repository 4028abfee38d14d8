"""GPU parity of the tcgen05 path (both tilings) against the oracle.

The skinny tiling splits the weight stream evenly over the SMs, so tiles are
shared between CTAs and finished from fp32 partial slots; the shapes below
cover whole and split tiles, ragged K, ragged weight rows and token counts
on both sides of every token-tile width.
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


def _run(p, tp, plan, max_tokens=None):
    A, Bs = p.shards(tp)
    Ad = [dev(a, "bf16") for a in A]
    Bd = [dev(b, "bf16") for b in Bs]
    m = B().TpMlp(p.d_in, p.d_ff, tp, p.act, "bf16", max_tokens or p.tokens, d_out=p.d_out)
    m.set_plan(plan)
    packed = m.pack(Ad, Bd)
    out = m.forward_packed(dev(p.x, "bf16"), packed)
    torch.cuda.synchronize()
    B().tp_mlp_get_device_status(m.h)
    return m, out, A, Bs, packed


def test_tc_first_small_case():
    """One small skinny case and one small wide case, run first."""
    p = inputs.generate(8, 256, 512, "swiglu", "bf16", seed=1, init="fan_in", d_out=256)
    A, Bs = p.shards(2)
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, "swiglu")
    for plan in ("tc_skinny", "tc_wide"):
        m, out, _, _, _ = _run(p, 2, plan)
        assert m.last_plan == plan
        assert_close(out, ref, "bf16", plan)


@pytest.mark.parametrize("plan,T", [("tc_skinny", 1), ("tc_skinny", 16), ("tc_skinny", 33),
                                    ("tc_wide", 1), ("tc_wide", 130)])
def test_tc_integer_exact(plan, T):
    """Small integers: tensor-core fp32 sums are exact, so the only rounding is
    the final bf16 one -> GPU == round_to_bf16(oracle) bit for bit."""
    p = inputs.integer_inputs(T, 64, 256, 264, "identity", seed=T, lo=-1, hi=1)
    A, Bs = p.shards(4)
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, "identity")
    _, out, _, _, _ = _run(p, 4, plan)
    assert np.array_equal(out.float().cpu().numpy(), inputs.round_to_bf16(ref.astype(np.float32)))


SHAPES = [  # (d_in, d_ff, d_out, tp)
    (512, 1024, 384, 4),
    (520, 384, 264, 2),     # ragged K (not a multiple of 64) and ragged output rows
    (4096, 1024, 256, 8),   # long K: tiles split across CTAs
    (256, 8192, 512, 8),    # long second projection K
]


@pytest.mark.parametrize("act", ["swiglu", "tanh", "identity"])
@pytest.mark.parametrize("T", [1, 5, 16, 17, 32, 33, 64, 100, 128])
@pytest.mark.parametrize("shape", SHAPES)
def test_tc_skinny_parity(act, T, shape):
    d, f, dout, tp = shape
    p = inputs.generate(T, d, f, act, "bf16", seed=T + f, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, act)
    m, out, _, _, packed = _run(p, tp, "tc_skinny")
    assert m.last_plan == "tc_skinny"
    assert_close(out, ref, "bf16", f"skinny T={T}")
    again = m.forward_packed(dev(p.x, "bf16"), packed)   # tile counters were reset
    assert torch.equal(out, again)


@pytest.mark.parametrize("act", ["swiglu", "tanh"])
@pytest.mark.parametrize("T", [5, 32, 100, 128])
@pytest.mark.parametrize("shape", SHAPES)
def test_tc_skinny_split_finish_modes_agree(act, T, shape):
    """Split tiles finished by the last CTA inside the GEMM, or by the reduction
    kernel behind it.  On packed weights the reduction route also uses 128-row
    tiles where it can (the in-kernel fixup keeps 256), so the split points
    differ and the oracle decides; the shard-form test below, where both
    routes tile alike, checks that they agree bit for bit."""
    d, f, dout, tp = shape
    p = inputs.generate(T, d, f, act, "bf16", seed=7 * T + f, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, act)
    m = B().TpMlp(d, f, tp, act, "bf16", T, d_out=dout)
    m.set_plan("tc_skinny")
    packed = m.pack([dev(a, "bf16") for a in A], [dev(b, "bf16") for b in Bs])
    x = dev(p.x, "bf16")
    outs = {}
    for mode in ("in_kernel", "separate", "in_kernel"):
        m.set_splitk(mode)
        out = m.forward_packed(x, packed)
        torch.cuda.synchronize()
        B().tp_mlp_get_device_status(m.h)
        assert_close(out, ref, "bf16", f"skinny {mode} T={T}")
        # every tile of these shapes is split: one reduction kernel per projection
        assert m.last_launches == (4 if mode == "separate" else 2)
        if mode in outs:
            assert torch.equal(out, outs[mode])     # counters were left at zero
        outs[mode] = out
    assert set(outs) == {"in_kernel", "separate"}



@pytest.mark.parametrize("api", ["packed", "shard"])
@pytest.mark.parametrize("T", [40, 100])
def test_tc_skinny_whole_128_row_tiles(api, T):
    """About as many 128-row tiles as SMs (packed weights): each CTA takes one
    whole first-projection tile (no partial slots, no reduction kernel); the
    second projection's few tiles are split evenly, every CTA inside one tile.
    The shard form keeps 256-row tiles, split evenly in two."""
    d, f, dout, tp = 256, 16384, 512, 8
    p = inputs.generate(T, d, f, "tanh", "bf16", seed=T + 5, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, "tanh")
    m = B().TpMlp(d, f, tp, "tanh", "bf16", T, d_out=dout)
    m.set_plan("tc_skinny")
    Ad, Bd = [dev(a, "bf16") for a in A], [dev(b, "bf16") for b in Bs]
    if api == "packed":
        out = m.forward_packed(dev(p.x, "bf16"), m.pack(Ad, Bd))
    else:
        out = m.forward(dev(p.x, "bf16"), Ad, Bd)
    torch.cuda.synchronize()
    B().tp_mlp_get_device_status(m.h)
    assert_close(out, ref, "bf16", f"whole 128-row tiles {api} T={T}")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if api == "packed" and 5 * 128 >= 4 * sms and 128 <= sms:   # 128 first-projection tiles fit the rule
        assert m.last_launches == 3                 # GEMM, GEMM + reduction


@pytest.mark.parametrize("act", ["swiglu", "tanh"])
@pytest.mark.parametrize("T", [1, 127, 128, 129, 300, 1000])
@pytest.mark.parametrize("shape", SHAPES[:3])
def test_tc_wide_parity(act, T, shape):
    d, f, dout, tp = shape
    p = inputs.generate(T, d, f, act, "bf16", seed=T + d, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    rows = p.sample_rows(64)
    ref = oracle.tp_mlp_sharded(p.x[rows], A, Bs, act)
    m, out, _, _, _ = _run(p, tp, "tc_wide")
    assert m.last_plan == "tc_wide"
    assert_close(out[torch.from_numpy(rows).cuda()], ref, "bf16", f"wide T={T}")


def test_auto_plan_uses_tensor_cores():
    p = inputs.generate(300, 256, 512, "swiglu", "bf16", seed=2)
    A, Bs = p.shards(2)
    m = B().TpMlp(256, 512, 2, "swiglu", "bf16", max_tokens=300)
    packed = m.pack([dev(a, "bf16") for a in A], [dev(b, "bf16") for b in Bs])
    x = dev(p.x, "bf16")
    m.forward_packed(x[:32], packed)
    assert m.last_plan == "tc_fused"
    m.forward_packed(x, packed)
    assert m.last_plan == "tc_wide"
    m.forward_packed(x[:2], packed)
    assert m.last_plan == "tc_fused"
    m.set_plan("tc")                   # tensor cores, tiling by token count
    m.forward_packed(x[:2], packed)
    assert m.last_plan == "tc_fused"
    m.set_plan("auto")
    m.forward_packed(x[:1], packed)
    assert m.last_plan == "gemv"


@pytest.mark.parametrize("act", ["swiglu", "tanh"])
@pytest.mark.parametrize("T", [1, 255, 256, 257, 600, 2100])
@pytest.mark.parametrize("shape", SHAPES[:3])
def test_tc_wide256_parity(act, T, shape):
    """256-token tiles (two M=128 MMAs per weight tile, one TMEM buffer)."""
    d, f, dout, tp = shape
    p = inputs.generate(T, d, f, act, "bf16", seed=T + 7 * d, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    rows = p.sample_rows(64)
    ref = oracle.tp_mlp_sharded(p.x[rows], A, Bs, act)
    m, out, _, _, _ = _run(p, tp, "tc_wide256")
    assert m.last_plan == "tc_wide256"
    assert_close(out[torch.from_numpy(rows).cuda()], ref, "bf16", f"wide256 T={T}")


@pytest.mark.parametrize("plan", ["tc_pair", "tc_pair2"])
@pytest.mark.parametrize("act", ["swiglu", "tanh", "identity"])
@pytest.mark.parametrize("T", [1, 100, 255, 256, 257, 600, 2100])
@pytest.mark.parametrize("shape", SHAPES[:3])
def test_tc_pair_parity(plan, act, T, shape):
    """Pairs of CTAs (cta_group::2 MMAs): 256 tokens x 256 weight rows per pair
    with two TMEM accumulators per CTA (tc_pair), or 256 x 512 with two weight
    tiles per X stage (tc_pair2; an odd tile count leaves the last unit half
    empty); ragged token and weight tails."""
    d, f, dout, tp = shape
    p = inputs.generate(T, d, f, act, "bf16", seed=T + 13 * d, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    rows = p.sample_rows(64)
    ref = oracle.tp_mlp_sharded(p.x[rows], A, Bs, act)
    m, out, _, _, _ = _run(p, tp, plan)
    assert m.last_plan == plan
    assert_close(out[torch.from_numpy(rows).cuda()], ref, "bf16", f"{plan} T={T}")


@pytest.mark.parametrize("plan", ["tc_pair", "tc_pair2"])
@pytest.mark.parametrize("T", [3, 300, 1030])
def test_tc_pair_integer_exact(plan, T):
    p = inputs.integer_inputs(T, 64, 512, 264, "identity", seed=T + 5, lo=-1, hi=1)
    m, out, A, Bs, _ = _run(p, 4, plan)
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, "identity")
    assert np.array_equal(out.float().cpu().numpy(), inputs.round_to_bf16(ref.astype(np.float32)))


def test_tc_pair_agrees_with_wide256():
    """The pair tiling and the 1-CTA 256-token tiling add the same products in the
    same k order; they agree within the bf16 bound (and with the oracle)."""
    p = inputs.generate(700, 512, 2048, "swiglu", "bf16", seed=77, init=0.02)
    outs = []
    for plan in ("tc_pair", "tc_pair2", "tc_wide256"):
        _, out, _, _, _ = _run(p, 4, plan)
        outs.append(out)
    assert_close(outs[0], outs[2].float().cpu().numpy(), "bf16", "pair vs wide256")
    assert_close(outs[1], outs[2].float().cpu().numpy(), "bf16", "pair2 vs wide256")


FUSED_SHAPES = SHAPES + [
    (512, 16384, 512, 8),   # 128 first-projection tiles of 128 rows: one whole tile per CTA
]


@pytest.mark.parametrize("act", ["swiglu", "tanh", "identity"])
@pytest.mark.parametrize("T", [1, 5, 17, 33, 100, 128])
@pytest.mark.parametrize("shape", FUSED_SHAPES)
def test_tc_fused_parity(act, T, shape):
    """Both skinny projections in one persistent launch: the second projection's
    H loads wait on a device count of stored first-projection tiles (whole
    tiles, or split tiles finished inside the kernel by their last CTA).  The
    last CTA resets the count, so repeated calls agree bit for bit."""
    d, f, dout, tp = shape
    p = inputs.generate(T, d, f, act, "bf16", seed=3 * T + f, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, act)
    m, out, _, _, packed = _run(p, tp, "tc_fused")
    assert m.last_plan == "tc_fused"
    assert_close(out, ref, "bf16", f"fused T={T}")
    x = dev(p.x, "bf16")
    for _ in range(3):
        assert torch.equal(m.forward_packed(x, packed), out)
    torch.cuda.synchronize()
    B().tp_mlp_get_device_status(m.h)


@pytest.mark.parametrize("T", [3, 33, 128])
def test_tc_fused_integer_exact(T):
    p = inputs.integer_inputs(T, 64, 256, 264, "identity", seed=T + 9, lo=-1, hi=1)
    m, out, A, Bs, _ = _run(p, 4, "tc_fused")
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, "identity")
    assert np.array_equal(out.float().cpu().numpy(), inputs.round_to_bf16(ref.astype(np.float32)))


def test_tc_fused_token_counts_and_graph_replay():
    """Calls of different token counts in turn on one handle, then the same
    calls captured in a CUDA graph and replayed with new inputs: the counters
    the kernel waits on live on the device and come back to zero after every
    launch."""
    d, f, dout, tp = 1024, 4096, 1024, 4
    Ts = (64, 7, 33)
    m = B().TpMlp(d, f, tp, "swiglu", "bf16", max(Ts), d_out=dout)
    m.set_plan("tc_fused")
    p = inputs.generate(max(Ts), d, f, "swiglu", "bf16", seed=21, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    packed = m.pack([dev(a, "bf16") for a in A], [dev(b, "bf16") for b in Bs])
    x = dev(p.x, "bf16")
    for T in Ts + Ts[:1]:
        out = m.forward_packed(x[:T], packed)
        assert m.last_plan == "tc_fused"
        assert_close(out, oracle.tp_mlp_sharded(p.x[:T], A, Bs, "swiglu"), "bf16", f"fused T={T}")
    outs = [torch.empty(T, dout, dtype=torch.bfloat16, device="cuda") for T in Ts]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for o, T in zip(outs, Ts):
            m.forward_packed(x[:T], packed, out=o)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for o, T in zip(outs, Ts):
            m.forward_packed(x[:T], packed, out=o)
    for step in range(2):
        q = inputs.generate(max(Ts), d, f, "swiglu", "bf16", seed=40 + step, init="fan_in", d_out=dout)
        x.copy_(dev(q.x, "bf16"))
        torch.cuda.synchronize()
        with torch.cuda.stream(s):
            g.replay()
        s.synchronize()
        for o, T in zip(outs, Ts):
            assert_close(o, oracle.tp_mlp_sharded(q.x[:T], A, Bs, "swiglu"), "bf16", f"graph step {step} T={T}")
    B().tp_mlp_get_device_status(m.h)
    del g


def test_auto_plan_tiling_by_token_count():
    """Packed weights: 128-token tiles up to 511 tokens, pairs of CTAs from 512 to
    4096, two-tile pairs above; the shard form keeps 256-token tiles from 2048."""
    p = inputs.generate(4097, 256, 512, "swiglu", "bf16", seed=3)
    A, Bs = p.shards(2)
    Ad, Bd = [dev(a, "bf16") for a in A], [dev(b, "bf16") for b in Bs]
    m = B().TpMlp(256, 512, 2, "swiglu", "bf16", max_tokens=4097)
    packed = m.pack(Ad, Bd)
    x = dev(p.x, "bf16")
    for T, plan in ((511, "tc_wide"), (512, "tc_pair"), (4096, "tc_pair"), (4097, "tc_pair2")):
        m.forward_packed(x[:T], packed)
        assert m.last_plan == plan, (T, m.last_plan)
    for T, plan in ((2047, "tc_wide"), (2048, "tc_wide256")):
        m.forward(x[:T], Ad, Bd)
        assert m.last_plan == plan, (T, m.last_plan)


# --- the shard form read directly by the tensor cores (MN-major weight operand) ---

RAW_SHAPES = [  # (d_in, d_ff, d_out, tp); f_s = d_ff / tp is a multiple of 64
    (512, 1024, 384, 4),
    (520, 384, 264, 2),     # ragged K and output width; f_s = 192: a rank's last tile is part padding
    (4096, 1024, 256, 8),   # long K, split tiles
    (256, 8192, 512, 8),    # long second-projection K over 8 ranks
]


def _run_shard_form(p, tp, plan, max_tokens=None):
    A, Bs = p.shards(tp)
    m = B().TpMlp(p.d_in, p.d_ff, tp, p.act, "bf16", max_tokens or p.tokens, d_out=p.d_out)
    m.set_plan(plan)
    out = m.forward(dev(p.x, "bf16"), [dev(a, "bf16") for a in A], [dev(b, "bf16") for b in Bs])
    torch.cuda.synchronize()
    B().tp_mlp_get_device_status(m.h)
    return m, out, A, Bs


@pytest.mark.parametrize("act", ["swiglu", "tanh", "identity"])
@pytest.mark.parametrize("plan,T", [("tc_skinny", 1), ("tc_skinny", 5), ("tc_skinny", 33), ("tc_skinny", 128),
                                    ("tc_wide", 129), ("tc_wide", 300), ("tc_wide256", 300), ("auto", 2)])
@pytest.mark.parametrize("shape", RAW_SHAPES)
def test_tc_shard_form_parity(act, plan, T, shape):
    d, f, dout, tp = shape
    p = inputs.generate(T, d, f, act, "bf16", seed=T + 3 * f + dout, init="fan_in", d_out=dout)
    m, out, A, Bs = _run_shard_form(p, tp, plan)
    assert m.last_plan == (plan if plan != "auto" else "tc_skinny")
    rows = p.sample_rows(64)
    ref = oracle.tp_mlp_sharded(p.x[rows], A, Bs, act)
    assert_close(out[torch.from_numpy(rows).cuda()], ref, "bf16", f"shard form {plan} T={T}")


@pytest.mark.parametrize("act", ["swiglu", "tanh", "identity"])
@pytest.mark.parametrize("T", [1, 5, 33, 100, 128])
@pytest.mark.parametrize("shape", RAW_SHAPES)
def test_tc_fused_shard_form_parity(act, T, shape):
    """The fused kernel on the per-rank shards (MN-major weight boxes, 256-row
    tiles, first-projection split tiles finished in the kernel), chosen
    explicitly; repeated calls agree bit for bit."""
    d, f, dout, tp = shape
    p = inputs.generate(T, d, f, act, "bf16", seed=7 * T + f + dout, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, act)
    m = B().TpMlp(d, f, tp, act, "bf16", T, d_out=dout)
    Ad, Bd = [dev(a, "bf16") for a in A], [dev(b, "bf16") for b in Bs]
    x = dev(p.x, "bf16")
    m.set_plan("tc_fused")
    out = m.forward(x, Ad, Bd)
    assert m.last_plan == "tc_fused"
    assert_close(out, ref, "bf16", f"fused shard form T={T}")
    for _ in range(2):
        assert torch.equal(m.forward(x, Ad, Bd), out)
    m.set_plan("tc_skinny")                     # the two-kernel tiling agrees with the oracle too
    assert_close(m.forward(x, Ad, Bd), ref, "bf16", f"skinny shard form T={T}")
    torch.cuda.synchronize()
    B().tp_mlp_get_device_status(m.h)


@pytest.mark.parametrize("T", [9, 64, 128])
def test_tc_shard_form_split_finish_modes_agree(T):
    d, f, dout, tp = RAW_SHAPES[0]
    p = inputs.generate(T, d, f, "swiglu", "bf16", seed=T + 11, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    Ad, Bd = [dev(a, "bf16") for a in A], [dev(b, "bf16") for b in Bs]
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, "swiglu")
    m = B().TpMlp(d, f, tp, "swiglu", "bf16", T, d_out=dout)
    m.set_plan("tc_skinny")
    outs = []
    for mode in ("in_kernel", "separate"):
        m.set_splitk(mode)
        outs.append(m.forward(dev(p.x, "bf16"), Ad, Bd))
        torch.cuda.synchronize()
        B().tp_mlp_get_device_status(m.h)
        assert_close(outs[-1], ref, "bf16", f"shard form {mode} T={T}")
    # the shard form keeps 256-row tiles on both routes: same split, same order
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("plan,T", [("tc_skinny", 3), ("tc_wide", 130), ("tc_wide256", 257)])
def test_tc_shard_form_integer_exact(plan, T):
    p = inputs.integer_inputs(T, 64, 512, 264, "identity", seed=T + 1, lo=-1, hi=1)
    _, out, A, Bs = _run_shard_form(p, 4, plan)
    ref = oracle.tp_mlp_sharded(p.x, A, Bs, "identity")
    assert np.array_equal(out.float().cpu().numpy(), inputs.round_to_bf16(ref.astype(np.float32)))


# --- per-rank partials on the tensor cores (each rank's K loop kept apart) ---

@pytest.mark.parametrize("act", ["swiglu", "tanh"])
@pytest.mark.parametrize("plan,T", [("tc_skinny", 1), ("tc_skinny", 5), ("tc_skinny", 33), ("tc_skinny", 128),
                                    ("tc_wide", 129), ("tc_wide", 300), ("tc_wide256", 300), ("auto", 7)])
@pytest.mark.parametrize("shape", RAW_SHAPES)
def test_tc_partials_parity(act, plan, T, shape):
    """Each rank's fp32 partial Z_i = act(X A_i) B_i against the oracle's, and
    their sum against the oracle's output and the forward on the same plan."""
    d, f, dout, tp = shape
    p = inputs.generate(T, d, f, act, "bf16", seed=T + 5 * f + dout, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    Ad, Bd = [dev(a, "bf16") for a in A], [dev(b, "bf16") for b in Bs]
    m = B().TpMlp(d, f, tp, act, "bf16", T, d_out=dout)
    m.set_plan(plan)
    x = dev(p.x, "bf16")
    gp = m.partials(x, Ad, Bd)
    torch.cuda.synchronize()
    B().tp_mlp_get_device_status(m.h)
    assert m.last_plan == (plan if plan != "auto" else "tc_skinny")
    assert gp.dtype == torch.float32 and gp.shape == (tp, T, dout)
    rows = p.sample_rows(64)
    ref, parts = oracle.tp_mlp_sharded(p.x[rows], A, Bs, act, return_partials=True)
    r = torch.from_numpy(rows).cuda()
    for i in range(tp):
        assert_close(gp[i][r], parts[i], "bf16", f"partial {i} {plan} T={T}")
    total = gp.sum(0)
    assert_close(total[r], ref, "bf16", f"sum of partials {plan} T={T}")
    out = m.forward(x, Ad, Bd)
    assert_close(out, total.cpu().numpy(), "bf16", f"forward vs sum of partials {plan} T={T}")


@pytest.mark.parametrize("plan,T", [("tc_skinny", 3), ("tc_skinny", 100), ("tc_wide", 130), ("tc_wide256", 257)])
def test_tc_partials_integer_exact(plan, T):
    """Small integers: every partial is exact in fp32, so each equals the
    oracle's partial bit for bit (split tiles included: the sums stay exact)."""
    p = inputs.integer_inputs(T, 64, 4 * 256, 264, "identity", seed=T + 2, lo=-1, hi=1)
    A, Bs = p.shards(4)
    m = B().TpMlp(64, 4 * 256, 4, "identity", "bf16", T, d_out=264)
    m.set_plan(plan)
    gp = m.partials(dev(p.x, "bf16"), [dev(a, "bf16") for a in A], [dev(b, "bf16") for b in Bs])
    torch.cuda.synchronize()
    assert m.last_plan == plan
    _, parts = oracle.tp_mlp_sharded(p.x, A, Bs, "identity", return_partials=True)
    assert np.array_equal(gp.cpu().numpy().astype(np.float64), np.asarray(parts))


# --- split tiles added across a thread-block cluster (distributed shared memory) ---

@pytest.mark.parametrize("act", ["tanh", "swiglu"])
@pytest.mark.parametrize("T", [5, 16, 33, 100, 128])
def test_tc_skinny_cluster_route_matches_reduction_kernel(act, T):
    """32 weight tiles per projection on 148 SMs: 4 CTAs share each tile.  The
    cluster route adds their slots across a cluster of 4 (two launches, no
    reduction kernel); it must give the reduction kernel's bits."""
    d, f, dout, tp = 512, 4096, 4096, 4
    p = inputs.generate(T, d, f, act, "bf16", seed=T + 17, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    Ad, Bd = [dev(a, "bf16") for a in A], [dev(b, "bf16") for b in Bs]
    m = B().TpMlp(d, f, tp, act, "bf16", T, d_out=dout)
    m.set_plan("tc_skinny")
    packed = m.pack(Ad, Bd)
    x = dev(p.x, "bf16")
    outs, launches = {}, {}
    for mode in ("cluster", "separate", "auto"):
        m.set_splitk(mode)
        outs[mode] = m.forward_packed(x, packed)
        torch.cuda.synchronize()
        B().tp_mlp_get_device_status(m.h)
        launches[mode] = m.last_launches
    assert launches["cluster"] < launches["separate"] == launches["auto"], launches
    assert torch.equal(outs["cluster"], outs["separate"])
    assert torch.equal(outs["auto"], outs["separate"])
    rows = p.sample_rows(32)
    assert_close(outs["cluster"][torch.from_numpy(rows).cuda()], oracle.tp_mlp_sharded(p.x[rows], A, Bs, act),
                 "bf16", f"cluster route T={T}")


@pytest.mark.parametrize("T", [3, 64])
def test_tc_cluster_route_shard_form_and_partials(T):
    """The shard form (256-row tiles) and the per-rank partials take the cluster
    route too: 32 tiles on 148 SMs.  Same bits as the reduction kernel."""
    d, f, dout, tp = 256, 2048, 8192, 2
    p = inputs.generate(T, d, f, "swiglu", "bf16", seed=T + 29, init="fan_in", d_out=dout)
    A, Bs = p.shards(tp)
    Ad, Bd = [dev(a, "bf16") for a in A], [dev(b, "bf16") for b in Bs]
    m = B().TpMlp(d, f, tp, "swiglu", "bf16", T, d_out=dout)
    m.set_plan("tc_skinny")
    x = dev(p.x, "bf16")
    res = {}
    for mode in ("cluster", "separate"):
        m.set_splitk(mode)
        out = m.forward(x, Ad, Bd)
        n_fwd = m.last_launches
        parts = m.partials(x, Ad, Bd)
        torch.cuda.synchronize()
        B().tp_mlp_get_device_status(m.h)
        res[mode] = (out, parts, n_fwd, m.last_launches)
    assert torch.equal(res["cluster"][0], res["separate"][0])
    assert torch.equal(res["cluster"][1], res["separate"][1])
    assert res["cluster"][2] < res["separate"][2] and res["cluster"][3] < res["separate"][3]
    ref, parts = oracle.tp_mlp_sharded(p.x, A, Bs, "swiglu", return_partials=True)
    assert_close(res["cluster"][0], ref, "bf16", "cluster route, shard form")
    for i in range(tp):
        assert_close(res["cluster"][1][i], parts[i], "bf16", f"cluster route, partial {i}")


def test_shard_form_falls_back_when_ranks_are_not_64_aligned():
    p = inputs.generate(4, 128, 8 * 40, "tanh", "bf16", seed=1)     # f_s = 40
    m, out, A, Bs = _run_shard_form(p, 8, "auto")
    assert m.last_plan == "simt"
    assert_close(out, oracle.tp_mlp_sharded(p.x, A, Bs, "tanh"), "bf16", "simt fallback")
