"""GPU parity of the fused all-reduce + residual add + RMSNorm against the oracle.

"7.4 推理侧并行", §7.4.2, optimisation 2: the residual add and RMSNorm that
follow the tensor-parallel all-reduce, fused into it.  The shapes cover one
CTA per row and rows split over clusters of 2..8 CTAs, widths that are not a
multiple of the block's 1024-element stride, the widest row the kernel takes,
in-place residual updates and the chain from tp_mlp_partials.
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


def _case(P, T, d, dtype, seed, scale=1.0):
    r = np.random.default_rng(seed)
    part = (r.standard_normal((P, T, d)) * scale).astype(np.float32)
    res = (r.standard_normal((T, d)) * scale).astype(np.float32)
    gamma = (1.0 + 0.1 * r.standard_normal(d)).astype(np.float32)
    if dtype == "bf16":
        res, gamma = inputs.round_to_bf16(res), inputs.round_to_bf16(gamma)
    return part, res, gamma


def _run(part, res, gamma, eps, dtype, in_place=False):
    p = torch.from_numpy(part).cuda()
    r = dev(res, dtype)
    g = dev(gamma, dtype)
    y, ro = B().tp_mlp_allreduce_residual_rmsnorm(p, r, g, eps, residual_out=r if in_place else None)
    torch.cuda.synchronize()
    return y, ro


SHAPES = [  # (P, T, d): CTAs per row follow from T and d
    (1, 1, 4),
    (2, 3, 64),
    (4, 5, 1000),       # 250 float4 groups: ragged against the 256-thread stride
    (8, 32, 8192),      # decode batch 32 at d_model 8192: 8-CTA clusters
    (8, 300, 2048),     # enough rows for one CTA per row
    (3, 1, 49152),      # the widest row
    (2, 150, 4100),     # 2-CTA clusters with a ragged last chunk
]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("P,T,d", SHAPES)
def test_fused_norm_parity(P, T, d, dtype):
    part, res, gamma = _case(P, T, d, dtype, seed=P * 1000 + T + d)
    eps = 1e-5
    y_ref, h_ref = oracle.allreduce_residual_rmsnorm(part, res, gamma, eps)
    y, ro = _run(part, res, gamma, eps, dtype)
    assert_close(y, y_ref, dtype, f"y P={P} T={T} d={d}")
    assert_close(ro, h_ref, dtype, f"residual P={P} T={T} d={d}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fused_norm_updates_the_residual_in_place(dtype):
    part, res, gamma = _case(4, 16, 8192, dtype, seed=5)
    y_ref, h_ref = oracle.allreduce_residual_rmsnorm(part, res, gamma, 1e-6)
    y, ro = _run(part, res, gamma, 1e-6, dtype, in_place=True)
    assert_close(y, y_ref, dtype, "y in place")
    assert_close(ro, h_ref, dtype, "residual in place")


def test_fused_norm_zero_rows_and_large_eps():
    """A zero row stays zero (eps > 0); a large eps damps the scale as the formula says."""
    part, res, gamma = _case(2, 4, 256, "f32", seed=6)
    part[:, 1, :] = 0.0
    res[1, :] = 0.0
    for eps in (1e-6, 10.0):
        y_ref, _ = oracle.allreduce_residual_rmsnorm(part, res, gamma, eps)
        y, _ = _run(part, res, gamma, eps, "f32")
        assert torch.all(y[1] == 0)
        assert_close(y, y_ref, "f32", f"eps={eps}")


def test_fused_norm_no_tokens_is_a_no_op():
    p = torch.zeros(2, 0, 64, device="cuda")
    r = torch.zeros(0, 64, device="cuda")
    g = torch.ones(64, device="cuda")
    y, ro = B().tp_mlp_allreduce_residual_rmsnorm(p, r, g, 1e-5)
    assert y.shape == (0, 64) and ro.shape == (0, 64)


def test_fused_norm_after_the_gpu_partials():
    """The chain a TP layer runs: every rank's Z_i (tp_mlp_partials on the GPU),
    then the fused all-reduce + residual + norm; against the oracle chain."""
    T, d, f, tp = 8, 256, 1024, 4
    p = inputs.generate(T, d, f, "tanh", "f32", seed=7, init="fan_in")
    A, Bs = p.shards(tp)
    parts_ref = oracle.tp_mlp_partials(p.x, A, Bs, "tanh")
    m = B().TpMlp(d, f, tp, "tanh", "f32", T)
    parts = m.partials(dev(p.x, "f32"), [dev(a, "f32") for a in A], [dev(b, "f32") for b in Bs])
    torch.cuda.synchronize()
    res = np.random.default_rng(8).standard_normal((T, d)).astype(np.float32)
    gamma = np.linspace(0.5, 1.5, d).astype(np.float32)
    y, ro = B().tp_mlp_allreduce_residual_rmsnorm(parts.contiguous(), dev(res, "f32"), dev(gamma, "f32"), 1e-5)
    torch.cuda.synchronize()
    # oracle chain in fp64 from the exact partials, then the fused step's definition
    h_ref = res.astype(np.float64) + parts_ref.sum(axis=0)
    rms = np.sqrt((h_ref ** 2).mean(axis=1, keepdims=True) + 1e-5)
    y_ref = h_ref / rms * gamma.astype(np.float64)
    assert_close(ro, h_ref, "f32", "residual after partials")
    assert_close(y, y_ref, "f32", "y after partials")
    # and the fused oracle on the GPU's own fp32 partials
    y2, h2 = oracle.allreduce_residual_rmsnorm(parts.cpu().numpy(), res, gamma, 1e-5)
    assert_close(y, y2, "f32", "y vs fused oracle")


def test_fused_norm_rejects_bad_arguments_before_launch():
    part, res, gamma = _case(2, 2, 64, "f32", seed=9)
    p = torch.from_numpy(part).cuda()
    r = dev(res, "f32")
    g = dev(gamma, "f32")
    L = B()._lib
    y = torch.empty_like(r)
    ptr = lambda t: B()._ptr(t)                                                  # noqa: E731
    assert L.tp_mlp_allreduce_residual_rmsnorm(ptr(p), 2, 2, 64, ptr(r), ptr(g), -1.0, 0, ptr(y), ptr(y), None) == 1
    assert L.tp_mlp_allreduce_residual_rmsnorm(ptr(p), 9, 2, 64, ptr(r), ptr(g), 0.0, 0, ptr(y), ptr(y), None) == 2
    assert L.tp_mlp_allreduce_residual_rmsnorm(ptr(p), 2, 2, 66, ptr(r), ptr(g), 0.0, 0, ptr(y), ptr(y), None) == 2
    # partials claimed larger than their allocation
    # (past the caching allocator's 2 MB segment, which is what the driver sees)
    assert L.tp_mlp_allreduce_residual_rmsnorm(ptr(p), 2, 100000, 64, ptr(r), ptr(g), 0.0, 0, ptr(y), ptr(y),
                                               None) == 2
    misaligned = B().ctypes.c_void_p(p.data_ptr() + 4)
    assert L.tp_mlp_allreduce_residual_rmsnorm(misaligned, 2, 1, 64, ptr(r), ptr(g), 0.0, 0, ptr(y), ptr(y),
                                               None) == 3


@pytest.mark.parametrize("name", ["fused_norm_decode_bs32", "fused_norm_prefill"])
def test_fused_norm_bench_configs_full_size(name):
    """The workloads bench.py times, at their full sizes; the prefill shape is
    checked on 256 seeded rows (the oracle handles rows independently)."""
    c = inputs.FUSED_NORM_CONFIGS[name]
    fi = inputs.generate_fused_norm(c["tokens"], c["d_model"], c["tp"], c["dtype"], c["seed"], c["eps"])
    y, ro = _run(fi.partials, fi.residual, fi.gamma, c["eps"], c["dtype"])
    rows = np.arange(c["tokens"])
    if c["tokens"] > 256:
        rows = np.sort(np.random.default_rng(c["seed"]).choice(c["tokens"], 256, replace=False))
    y_ref, h_ref = oracle.allreduce_residual_rmsnorm(fi.partials[:, rows], fi.residual[rows], fi.gamma, c["eps"])
    idx = torch.from_numpy(rows).cuda()
    assert_close(y[idx], y_ref, c["dtype"], f"{name} y")
    assert_close(ro[idx], h_ref, c["dtype"], f"{name} residual")
