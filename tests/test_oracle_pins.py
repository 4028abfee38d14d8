"""Pins for the oracle: each test ties it to something other than itself.

Sources (page title, section):
  [TP]   "LLM 推理并行化：先找瓶颈，再决定怎么切", §三 2) 张量并行（TP）
  [vLLM] "大模型推理系统揭秘（07）：Multi-GPU：一张卡不够时如何扩展？", §1.2.2–§1.2.4, §1.4.3
  [7.4]  "7.4 推理侧并行", §7.4.1

The pages' printed TP output [[-3.294438, 1.406896]] cannot pin anything: the
inputs that produced it are not printed ("parity unpinned" by that value).
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from tensor_sharded_mlp_b200 import counts, inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_counts.json")


def _rand(shape, seed, scale=1.0):
    r = np.random.default_rng(seed)
    return (r.standard_normal(shape) * scale).astype(np.float32)


def _problem(T, d, f, dout, act, seed):
    x = _rand((T, d), seed)
    if act == "swiglu":
        g = _rand((d, f), seed + 1, d ** -0.5)
        u = _rand((d, f), seed + 2, d ** -0.5)
        b = _rand((f, dout), seed + 3, f ** -0.5)
        return x, (g, u), b
    a = _rand((d, f), seed + 1, d ** -0.5)
    b = _rand((f, dout), seed + 3, f ** -0.5)
    return x, a, b


def _shard(a, b, act, P):
    f = b.shape[0]
    fs = f // P
    A, B = [], []
    for i in range(P):
        sl = slice(i * fs, (i + 1) * fs)
        if act == "swiglu":
            A.append(np.concatenate([a[0][:, sl], a[1][:, sl]], axis=1))
        else:
            A.append(a[:, sl])
        B.append(b[sl, :])
    return A, B


def _unsharded(x, a, b, act):
    if act == "swiglu":
        return oracle.tp_mlp_unsharded(x, a[0], b, act, a_up=a[1])
    return oracle.tp_mlp_unsharded(x, a, b, act)


# --- special cases that reduce to a library routine -------------------------

@pytest.mark.parametrize("P", [1, 2, 4])
@pytest.mark.parametrize("shape", [(3, 8, 8, 4), (5, 16, 12, 7), (1, 64, 32, 64)])
def test_identity_integer_exact(P, shape):
    """act = identity on small integers: every sum is an exact integer, so the
    oracle must equal numpy's int64 matmul chain bit for bit ([vLLM] §1.2.3)."""
    T, d, f, dout = shape
    if f % P:
        pytest.skip("uneven split")
    p = inputs.integer_inputs(T, d, f, dout, "identity", seed=11 + P)
    xi, ai, bi = (m.astype(np.int64) for m in (p.x, p.a, p.b))
    exact = (xi @ ai @ bi).astype(np.float64)
    A, B = p.shards(P)
    z, parts = oracle.tp_mlp_sharded(p.x, A, B, "identity", return_partials=True)
    assert np.array_equal(z, exact)
    assert np.array_equal(_unsharded(p.x, p.a, p.b, "identity"), exact)
    fs = f // P
    for i in range(P):
        sl = slice(i * fs, (i + 1) * fs)
        assert np.array_equal(parts[i], (xi @ ai[:, sl] @ bi[sl, :]).astype(np.float64))


@pytest.mark.parametrize("P", [1, 2])
def test_swiglu_integer_gate_zero_exact(P):
    """SwiGLU with gate = 0 gives SiLU(0) * up = 0 exactly, whatever up is."""
    p = inputs.integer_inputs(3, 8, 8, 5, "swiglu", seed=3)
    z = oracle.tp_mlp_unsharded(p.x, np.zeros_like(p.gate), p.b, "swiglu", a_up=p.up)
    assert np.array_equal(z, np.zeros_like(z))


def test_tanh_tp1_matches_numpy():
    """P = 1 is the plain MLP tanh(x @ A) @ B ([TP] worked function), here
    computed by numpy's float64 matmul and tanh."""
    x, a, b = _problem(5, 24, 40, 9, "tanh", 7)
    want = np.tanh(x.astype(np.float64) @ a.astype(np.float64)) @ b.astype(np.float64)
    got = oracle.tp_mlp_sharded(x, [a], [b], "tanh")
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


def test_swiglu_tp1_matches_torch():
    """P = 1 SwiGLU = (SiLU(x W1) * (x W3)) W2 ([vLLM] §1.4.3) with torch's float64
    silu and matmul as the library routine."""
    x, (g, u), b = _problem(4, 32, 48, 16, "swiglu", 9)
    tx, tg, tu, tb = (torch.from_numpy(m).double() for m in (x, g, u, b))
    want = ((torch.nn.functional.silu(tx @ tg) * (tx @ tu)) @ tb).numpy()
    A, B = _shard((g, u), b, "swiglu", 1)
    got = oracle.tp_mlp_sharded(x, A, B, "swiglu")
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)
    got2 = oracle.tp_mlp_unsharded(x, g, b, "swiglu", a_up=u)
    np.testing.assert_allclose(got2, want, rtol=1e-12, atol=1e-13)


# --- the column/row identity ([vLLM] §1.2.3 boxed equations) ------------------

@pytest.mark.parametrize("act", ["tanh", "swiglu", "identity"])
@pytest.mark.parametrize("P", [1, 2, 4, 8])
def test_sharded_equals_unsharded(act, P):
    x, a, b = _problem(6, 32, 64, 24, act, 100 + P)
    A, B = _shard(a, b, act, P)
    z = oracle.tp_mlp_sharded(x, A, B, act)
    ref = _unsharded(x, a, b, act)
    assert np.max(np.abs(z - ref)) <= 1e-12 * np.max(np.abs(ref))


@pytest.mark.parametrize("act", ["tanh", "swiglu"])
def test_partials_sum_and_slices(act):
    """Each partial is the unsharded MLP restricted to that rank's features, and
    the partials sum (in rank order) to the output."""
    P = 4
    x, a, b = _problem(3, 16, 32, 8, act, 21)
    A, B = _shard(a, b, act, P)
    z, parts = oracle.tp_mlp_sharded(x, A, B, act, return_partials=True)
    assert parts.shape == (P, 3, 8)
    acc = np.zeros_like(z)
    for i in range(P):
        acc = acc + parts[i]
    assert np.array_equal(acc, z)
    fs = 32 // P
    for i in range(P):
        sl = slice(i * fs, (i + 1) * fs)
        if act == "swiglu":
            ref = oracle.tp_mlp_unsharded(x, a[0][:, sl], b[sl], act, a_up=a[1][:, sl])
        else:
            ref = oracle.tp_mlp_unsharded(x, a[:, sl], b[sl], act)
        assert np.array_equal(parts[i], ref)


def test_page3_worked_shapes():
    """[vLLM] §1.2.3: X in R^{Bx8}; W1 8x8 split by columns into four 8x2; W2 8x4
    split by rows into four 2x4; Z = Z0+Z1+Z2+Z3 equals X W1 W2."""
    g = json.load(open(GOLDEN))["worked_split_shapes"]
    x, a, b = _problem(3, g["x_cols"], g["w1"][1], g["w2"][1], "identity", 5)
    assert a.shape == tuple(g["w1"]) and b.shape == tuple(g["w2"])
    A, B = _shard(a, b, "identity", g["tp"])
    assert all(s.shape == tuple(g["w1_shard"]) for s in A)
    assert all(s.shape == tuple(g["w2_shard"]) for s in B)
    z = oracle.tp_mlp_sharded(x, A, B, "identity")
    want = x.astype(np.float64) @ a.astype(np.float64) @ b.astype(np.float64)
    np.testing.assert_allclose(z, want, rtol=1e-13, atol=1e-14)
    assert z.shape == (3, 4)


# --- special values and closed forms ------------------------------------------

@pytest.mark.parametrize("act", ["tanh", "swiglu", "identity"])
def test_zero_input_gives_zero(act):
    _, a, b = _problem(2, 16, 16, 8, act, 1)
    A, B = _shard(a, b, act, 2)
    z = oracle.tp_mlp_sharded(np.zeros((2, 16), np.float32), A, B, act)
    assert np.array_equal(z, np.zeros_like(z))


def test_tanh_odd_symmetry():
    """tanh is odd and the projections are linear: Z(-X) = -Z(X) exactly."""
    x, a, b = _problem(4, 16, 32, 8, "tanh", 2)
    A, B = _shard(a, b, "tanh", 4)
    assert np.array_equal(oracle.tp_mlp_sharded(-x, A, B, "tanh"),
                          -oracle.tp_mlp_sharded(x, A, B, "tanh"))


def test_swiglu_up_is_linear_factor():
    """SiLU(gate) multiplies up: negating up negates Z exactly; negating gate does
    not (SiLU is not odd), which a sign slip in SiLU would break."""
    x, (g, u), b = _problem(3, 16, 16, 8, "swiglu", 4)
    z = oracle.tp_mlp_unsharded(x, g, b, "swiglu", a_up=u)
    assert np.array_equal(oracle.tp_mlp_unsharded(x, g, b, "swiglu", a_up=-u), -z)
    zg = oracle.tp_mlp_unsharded(x, -g, b, "swiglu", a_up=u)
    assert not np.allclose(zg, -z)


def test_scalar_closed_forms():
    """d_in = d_ff = d_out = 1.
    tanh:   z = b * tanh(x a); with a = atanh(1/2) (rounded to fp32), z ~ b / 2.
    SwiGLU: gate g = ln 3 gives sigma(g) = 3/4, so SiLU(ln 3) = (3/4) ln 3 and
            z = down * up * (3/4) ln 3 (x = 1, up = 2, down = 1 -> 1.5 ln 3)."""
    a = np.float32(math.atanh(0.5))
    z = oracle.tp_mlp_sharded(np.ones((1, 1), np.float32), [np.full((1, 1), a)],
                              [np.full((1, 1), 2.0, np.float32)], "tanh")
    assert abs(z[0, 0] - 2.0 * math.tanh(float(a))) < 1e-15
    assert abs(z[0, 0] - 1.0) < 1e-7
    g = np.float32(math.log(3.0))
    A = [np.array([[g, 2.0]], np.float32)]           # [gate | up]
    z = oracle.tp_mlp_sharded(np.ones((1, 1), np.float32), A,
                              [np.ones((1, 1), np.float32)], "swiglu")
    assert abs(z[0, 0] - 1.5 * math.log(3.0)) < 2e-7
    # SiLU(g) via scipy's logistic sigmoid, at the exact fp32 gate value
    assert abs(z[0, 0] - 2.0 * float(g) * scipy.special.expit(float(g))) < 1e-15


# --- brute force on tiny inputs -----------------------------------------------

def _brute(x, A, B, act):
    """Pure-Python loops; activation from the math module / scipy."""
    T, d = x.shape
    dout = B[0].shape[1]
    z = [[0.0] * dout for _ in range(T)]
    for Ai, Bi in zip(A, B):
        fs = Bi.shape[0]
        for t in range(T):
            for n in range(fs):
                s = sum(float(x[t, j]) * float(Ai[j, n]) for j in range(d))
                if act == "tanh":
                    h = math.tanh(s)
                elif act == "swiglu":
                    v = sum(float(x[t, j]) * float(Ai[j, fs + n]) for j in range(d))
                    h = s * float(scipy.special.expit(s)) * v
                else:
                    h = s
                for c in range(dout):
                    z[t][c] += h * float(Bi[n, c])
    return np.array(z)


@pytest.mark.parametrize("act", ["tanh", "swiglu", "identity"])
def test_brute_force_tiny(act):
    r = np.random.default_rng(77)
    for trial in range(12):
        T = int(r.integers(1, 6))
        d = int(r.integers(1, 10))
        P = int(r.choice([1, 2, 3, 4]))
        f = P * int(r.integers(1, 5))
        dout = int(r.integers(1, 7))
        x, a, b = _problem(T, d, f, dout, act, 1000 + trial)
        A, B = _shard(a, b, act, P)
        got = oracle.tp_mlp_sharded(x, A, B, act)
        want = _brute(x, A, B, act)
        assert np.max(np.abs(got - want)) <= 1e-12 * max(1.0, np.max(np.abs(want)))


# --- argument errors ----------------------------------------------------------

def test_shard_count_mismatch_is_an_error():
    """The worked function pairs shards strictly: unequal counts are an error."""
    x, a, b = _problem(1, 8, 8, 4, "tanh", 0)
    A, B = _shard(a, b, "tanh", 2)
    with pytest.raises(ValueError):
        oracle.tp_mlp_sharded(x, A, B[:1], "tanh")


def test_rejects_non_fp32_values():
    with pytest.raises(ValueError):
        oracle.tp_mlp_sharded(np.full((1, 1), 0.1), [np.ones((1, 1))], [np.ones((1, 1))])


# --- analytic counts ([7.4] §7.4.1) --------------------------------------------

@pytest.mark.parametrize("act", ["tanh", "swiglu"])
def test_mac_count_is_params_per_token(act):
    """The loops execute exactly N multiply-adds per token (2N FLOPs/token)."""
    T, d, f, dout, P = 3, 16, 32, 12, 4
    x, a, b = _problem(T, d, f, dout, act, 8)
    A, B = _shard(a, b, act, P)
    _, macs = oracle.tp_mlp_sharded(x, A, B, act, return_macs=True)
    N = counts.mlp_params(d, f, dout, act)
    assert N == sum(s.size for s in A) + sum(s.size for s in B)
    assert macs == T * N
    g = json.load(open(GOLDEN))["forward_flops_per_token_per_param"]["value"]
    assert counts.forward_flops(T, d, f, dout, act) == g * macs
