"""Pins for the oracle of the fused all-reduce + residual add + RMSNorm.

Source: "7.4 推理侧并行", §7.4.2, optimisation 2 (custom all-reduce): the
residual add and RMSNorm that follow the tensor-parallel all-reduce are fused
into it.  The pages print no numbers for this step, so every pin below ties the
oracle to a library routine, a closed form or the (separately pinned) MLP
oracle.  A dropped eps, a wrong divisor, a missing gamma or residual, a skipped
rank or a square root in the wrong place each fails at least one of them.
"""
import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32)


@pytest.mark.parametrize("P,T,d,eps", [(1, 1, 1, 0.0), (2, 3, 7, 1e-6), (8, 4, 64, 1e-5), (3, 2, 1000, 0.5)])
def test_matches_torch_rms_norm_in_float64(P, T, d, eps):
    """Library routine: torch.nn.functional.rms_norm on h = residual + sum of the
    partials (numpy's sum), all in float64."""
    p, r, g = _rand((P, T, d), 1), _rand((T, d), 2), _rand((d,), 3)
    y, h = oracle.allreduce_residual_rmsnorm(p, r, g, eps)
    h_ref = r.astype(np.float64) + p.astype(np.float64).sum(axis=0)
    y_ref = torch.nn.functional.rms_norm(torch.from_numpy(h_ref), (d,), weight=torch.from_numpy(g.astype(np.float64)),
                                         eps=eps).numpy()
    np.testing.assert_allclose(h, h_ref, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)


def test_unit_gain_rows_have_unit_mean_square():
    """gamma = 1, eps = 0: every nonzero output row has mean(y^2) = 1 exactly."""
    p, r = _rand((4, 6, 96), 4), _rand((6, 96), 5)
    y, _ = oracle.allreduce_residual_rmsnorm(p, r, np.ones(96, np.float32), 0.0)
    np.testing.assert_allclose((y ** 2).mean(axis=1), 1.0, rtol=1e-13)


def test_constant_row_closed_form():
    """A row whose h is the constant a: y_j = a / sqrt(a^2 + eps) * gamma_j."""
    d, a, eps = 10, -3.0, 0.25
    p = np.zeros((2, 1, d), np.float32)
    p[0, 0, :] = -1.0
    p[1, 0, :] = -2.5
    r = np.full((1, d), 0.5, np.float32)       # h = 0.5 - 1 - 2.5 = -3
    g = _rand((d,), 6)
    y, h = oracle.allreduce_residual_rmsnorm(p, r, g, eps)
    assert np.all(h == a)
    np.testing.assert_allclose(y[0], a / np.sqrt(a * a + eps) * g.astype(np.float64), rtol=1e-15)


def test_scale_invariance_without_eps():
    """With eps = 0 the norm ignores a positive scale of the row: y(c h) = y(h)."""
    p, r, g = _rand((3, 2, 50), 7), _rand((2, 50), 8), _rand((50,), 9)
    y1, _ = oracle.allreduce_residual_rmsnorm(p, r, g, 0.0)
    y2, _ = oracle.allreduce_residual_rmsnorm(4.0 * p, 4.0 * r, g, 0.0)   # powers of 2: exact
    np.testing.assert_allclose(y1, y2, rtol=1e-14)


def test_zero_row_stays_zero():
    p = np.zeros((2, 1, 8), np.float32)
    y, h = oracle.allreduce_residual_rmsnorm(p, np.zeros((1, 8), np.float32), _rand((8,), 10), 1e-6)
    assert np.all(y == 0.0) and np.all(h == 0.0)


def test_rank_sum_is_the_mlp_output():
    """Zero residual: h is the all-reduce of the MLP oracle's per-rank partials,
    i.e. the unsharded MLP (pinned on its own in test_oracle_pins.py)."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((3, 16)).astype(np.float32)
    a = (rng.standard_normal((16, 32)) * 0.25).astype(np.float32)
    b = (rng.standard_normal((32, 12)) * 0.2).astype(np.float32)
    P = 4
    parts = oracle.tp_mlp_partials(x, np.split(a, P, axis=1), np.split(b, P, axis=0), "tanh")
    # the partials are fp64; the fused step takes fp32 inputs, so compare against
    # the fp32-rounded partials' exact sum
    p32 = parts.astype(np.float32)
    _, h = oracle.allreduce_residual_rmsnorm(p32, np.zeros((3, 12), np.float32), np.ones(12, np.float32), 0.0)
    np.testing.assert_allclose(h, p32.astype(np.float64).sum(axis=0), rtol=1e-14)
    np.testing.assert_allclose(h, oracle.tp_mlp_unsharded(x, a, b, "tanh"), rtol=1e-6, atol=1e-6)


def test_argument_errors():
    p, r, g = _rand((2, 1, 4), 12), _rand((1, 4), 13), _rand((4,), 14)
    with pytest.raises(ValueError):
        oracle.allreduce_residual_rmsnorm(p, r, g, -1.0)
    with pytest.raises(ValueError):
        oracle.allreduce_residual_rmsnorm(p, r[:, :3], g, 0.0)
    with pytest.raises(ValueError):
        oracle.allreduce_residual_rmsnorm(p[0], r, g, 0.0)
