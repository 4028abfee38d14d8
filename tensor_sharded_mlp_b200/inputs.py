"""Seeded synthetic inputs for the tensor-parallel MLP.

This module is the one piece shared by the CUDA path's tests and benchmark and
by the oracle's tests: it draws numbers and slices them into per-rank shards.
It holds none of the MLP's arithmetic (no products, sums or activations).

Recipe (fixed, so every user of a config sees the same numbers):
  * ``numpy.random.default_rng(seed)``; ``standard_normal`` in float64, drawn in
    row-major order, full unsharded matrices, in the order
    X (T x d_in), then A (tanh / identity) or gate then up (SwiGLU, each
    d_in x d_ff), then B / down (d_ff x d_out).  Large matrices are drawn in row
    chunks; the stream is the same as one draw.
  * each matrix is scaled by its standard deviation: ``"fan_in"`` means
    variance 1/fan_in (std = fan_in**-0.5, fan_in = d_in for the first
    projection, d_ff for the second); a number is the std itself (0.02).  X is
    N(0, 1).
  * values are cast to fp32; for a bf16 config they are then rounded to bf16
    (round-to-nearest-even) and kept as fp32 arrays that hold the bf16 values
    exactly, so the oracle and the GPU see identical numbers.
  * a shard is a slice of the full matrix: rank i's first-projection block is
    columns [i*f_s, (i+1)*f_s) (for SwiGLU the gate block followed by the up
    block of the same columns), its second-projection block is rows
    [i*f_s, (i+1)*f_s).  So every TP degree computes the same function.
  * sampled rows (for checking very large token counts) are drawn from the same
    generator after the weights: ``rng.choice(T, n, replace=False)``, sorted.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
from typing import Optional

import numpy as np

_CHUNK_ELEMS = 1 << 24

# The workloads: shapes, dtypes, activation, initialisation and seed.
CONFIGS = {
    "tiny": dict(dtype="f32", act="tanh", tokens=4, d_model=64, d_ff=256, tp=2,
                 init="fan_in", seed=0),
    "decode_bs1": dict(dtype="bf16", act="swiglu", tokens=1, d_model=8192, d_ff=28672, tp=8,
                       init=0.02, seed=1),
    "decode_bs32": dict(dtype="bf16", act="swiglu", tokens=32, d_model=8192, d_ff=28672, tp=8,
                        init=0.02, seed=2),
    "sweep": dict(dtype="bf16", act="tanh", tokens=(1, 16, 128, 1024, 4096), d_model=4096,
                  d_ff=16384, tp=(1, 2, 4, 8), init="fan_in", seed=3),
    "prefill": dict(dtype="bf16", act="swiglu", tokens=8192, d_model=8192, d_ff=28672,
                    tp=(2, 4, 8), init=0.02, seed=4, sample_rows=256),
}


# The fused all-reduce + residual add + RMSNorm step ("7.4 推理侧并行" §7.4.2):
# P rank partials of the second projection's output, the residual stream and
# the norm's gain, at the decode batch-32 and prefill shapes of the MLP configs.
FUSED_NORM_CONFIGS = {
    "fused_norm_decode_bs32": dict(dtype="bf16", tokens=32, d_model=8192, tp=8, eps=1e-5, seed=21),
    "fused_norm_prefill": dict(dtype="bf16", tokens=8192, d_model=8192, tp=8, eps=1e-5, seed=22),
}


@dataclasses.dataclass
class FusedNormInputs:
    partials: np.ndarray   # P x T x d, fp32
    residual: np.ndarray   # T x d (dtype-representable values in fp32)
    gamma: np.ndarray      # d
    eps: float


def generate_fused_norm(tokens: int, d_model: int, tp: int, dtype: str, seed: int, eps: float = 1e-5
                        ) -> FusedNormInputs:
    """Seeded inputs of the fused step: rng(seed), float64 standard normals drawn
    in the order partials (P x T x d, N(0, 1), kept fp32), residual (T x d,
    N(0, 1)), gamma (d, 1 + 0.1 N(0, 1)); residual and gamma rounded to bf16 for
    a bf16 config."""
    rng = np.random.default_rng(seed)
    part = np.empty((tp, tokens, d_model), np.float32)
    for i in range(tp):
        part[i] = _draw(rng, tokens, d_model, 1.0, "f32")
    res = _draw(rng, tokens, d_model, 1.0, dtype)
    g = (1.0 + 0.1 * rng.standard_normal(d_model)).astype(np.float32)
    if dtype == "bf16":
        g = round_to_bf16(g)
    return FusedNormInputs(part, res, g, eps)


# Merging partial attention results across KV shards (decode context
# parallelism, "LLM 推理并行化" §三 4)): P ranks' per-row statistics for a
# decode batch of `tokens` queries over `heads` heads of `head_dim`, the head
# layout of the d_model 8192 configs (64 heads of 128).
ATTN_MERGE_CONFIGS = {
    "attn_merge_decode_bs32": dict(dtype="f32", tokens=32, heads=64, head_dim=128, tp=8, keys_per_rank=512,
                                   seed=31),
    "attn_merge_decode_bs256": dict(dtype="bf16", tokens=256, heads=64, head_dim=128, tp=8, keys_per_rank=512,
                                    seed=32),
}


@dataclasses.dataclass
class AttnMergeInputs:
    maximum: np.ndarray    # P x rows, fp32
    exp_sum: np.ndarray    # P x rows, fp32
    weighted: np.ndarray   # P x rows x head_dim (dtype-representable values in fp32)


def generate_attn_merge(tp: int, rows: int, head_dim: int, dtype: str, seed: int, keys_per_rank: int = 512
                        ) -> AttnMergeInputs:
    """Seeded per-rank statistics: rng(seed) draws, in order, the maxima
    (P x rows, N(0, 2^2)), the exponential sums (P x rows, 1 + U(0,1) *
    (keys_per_rank - 1): at least the maximum's own term, at most one per key)
    and the weighted sums (P x rows x head_dim, N(0, 1) * sqrt(exp_sum), a sum
    of that many unit-scale values); the weighted sums are rounded to bf16 for a
    bf16 config."""
    rng = np.random.default_rng(seed)
    m = (rng.standard_normal((tp, rows)) * 2.0).astype(np.float32)
    s = (1.0 + rng.random((tp, rows)) * (keys_per_rank - 1)).astype(np.float32)
    w = np.empty((tp, rows, head_dim), np.float32)
    for i in range(tp):
        w[i] = _draw(rng, rows, head_dim, 1.0, "f32") * np.sqrt(s[i])[:, None].astype(np.float32)
    if dtype == "bf16":
        w = round_to_bf16(w)
    return AttnMergeInputs(m, s, w)


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32 holding them.

    Works on the 32-bit patterns: adding 0x7FFF plus the lowest kept bit and
    clearing the low 16 bits rounds to nearest, ties to even.  For every finite
    input the sum stays below 2**32 (the largest finite pattern is 0xFF7FFFFF).
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32)
    lsb = (bits >> 16) & np.uint32(1)
    out = ((bits + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)).view(np.float32)
    # NaN/Inf never occur for finite normal draws; keep them untouched anyway.
    special = ~np.isfinite(a)
    if special.any():
        out = out.copy()
        out[special] = a[special]
    return out


def _std(init, fan_in: int) -> float:
    if init == "fan_in":
        return float(fan_in) ** -0.5
    return float(init)


def _draw(rng: np.random.Generator, rows: int, cols: int, std: float, dtype: str) -> np.ndarray:
    # The draws stay in one sequential stream; scaling, the fp32 cast and the
    # bf16 rounding of a chunk run on a worker thread while the next chunk is
    # drawn (numpy releases the GIL in both), which leaves the values unchanged.
    out = np.empty((rows, cols), dtype=np.float32)
    step = max(1, _CHUNK_ELEMS // max(cols, 1))

    def finish(r0, r1, chunk):
        v = (chunk * std).astype(np.float32)
        out[r0:r1] = round_to_bf16(v) if dtype == "bf16" else v

    with concurrent.futures.ThreadPoolExecutor(max_workers=2) as ex:
        pending = []
        for r0 in range(0, rows, step):
            r1 = min(rows, r0 + step)
            pending.append(ex.submit(finish, r0, r1, rng.standard_normal((r1 - r0, cols))))
            if len(pending) > 2:
                pending.pop(0).result()
        for f in pending:
            f.result()
    return out


@dataclasses.dataclass
class MlpInputs:
    """One seeded problem: X and the full (unsharded) weight matrices."""
    act: str
    dtype: str
    tokens: int
    d_in: int
    d_ff: int
    d_out: int
    seed: int
    x: np.ndarray
    a: Optional[np.ndarray]        # tanh / identity: d_in x d_ff
    gate: Optional[np.ndarray]     # SwiGLU: d_in x d_ff
    up: Optional[np.ndarray]       # SwiGLU: d_in x d_ff
    b: np.ndarray                  # d_ff x d_out
    rng: np.random.Generator       # continues after the weights (row sampling)

    def shards(self, tp: int):
        """Per-rank shards: (A_shards, B_shards), lists of fp32 arrays.

        tanh / identity: A_i = A[:, cols_i] (d_in x f_s).
        SwiGLU:          A_i = [gate[:, cols_i] | up[:, cols_i]] (d_in x 2 f_s).
        Always:          B_i = B[cols_i, :]  (f_s x d_out).
        """
        if tp < 1 or self.d_ff % tp:
            raise ValueError(f"d_ff={self.d_ff} is not divisible by tp={tp}")
        fs = self.d_ff // tp
        a_sh, b_sh = [], []
        for i in range(tp):
            sl = slice(i * fs, (i + 1) * fs)
            if self.act == "swiglu":
                a_sh.append(np.ascontiguousarray(np.concatenate(
                    [self.gate[:, sl], self.up[:, sl]], axis=1)))
            else:
                a_sh.append(np.ascontiguousarray(self.a[:, sl]))
            b_sh.append(np.ascontiguousarray(self.b[sl, :]))
        return a_sh, b_sh

    def sample_rows(self, n: int) -> np.ndarray:
        """n distinct token rows, drawn after the weights, sorted."""
        n = min(n, self.tokens)
        return np.sort(self.rng.choice(self.tokens, n, replace=False))


def generate(tokens: int, d_model: int, d_ff: int, act: str = "tanh", dtype: str = "f32",
             seed: int = 0, init="fan_in", d_out: Optional[int] = None) -> MlpInputs:
    """Draw one problem following the recipe in the module docstring."""
    if act not in ("tanh", "swiglu", "identity"):
        raise ValueError(f"unknown activation {act!r}")
    if dtype not in ("f32", "bf16"):
        raise ValueError(f"unknown dtype {dtype!r}")
    d_out = d_model if d_out is None else d_out
    rng = np.random.default_rng(seed)
    x = _draw(rng, tokens, d_model, 1.0, dtype)
    a = gate = up = None
    if act == "swiglu":
        gate = _draw(rng, d_model, d_ff, _std(init, d_model), dtype)
        up = _draw(rng, d_model, d_ff, _std(init, d_model), dtype)
    else:
        a = _draw(rng, d_model, d_ff, _std(init, d_model), dtype)
    b = _draw(rng, d_ff, d_out, _std(init, d_ff), dtype)
    return MlpInputs(act, dtype, tokens, d_model, d_ff, d_out, seed, x, a, gate, up, b, rng)


def generate_config(name: str, tokens: Optional[int] = None) -> MlpInputs:
    """The named workload; ``tokens`` picks one entry where the config lists several."""
    c = CONFIGS[name]
    t = c["tokens"]
    if isinstance(t, tuple):
        if tokens is None:
            raise ValueError(f"config {name} lists several token counts; pick one")
        t = tokens
    elif tokens is not None and tokens != t:
        raise ValueError(f"config {name} is defined for tokens={t}")
    return generate(t, c["d_model"], c["d_ff"], c["act"], c["dtype"], c["seed"], c["init"])


def integer_inputs(tokens: int, d_in: int, d_ff: int, d_out: int, act: str, seed: int,
                   lo: int = -4, hi: int = 4) -> MlpInputs:
    """Small-integer X and weights (exact in fp32, bf16 and fp64 sums)."""
    rng = np.random.default_rng(seed)
    def ints(r, c):
        return rng.integers(lo, hi + 1, size=(r, c)).astype(np.float32)
    x = ints(tokens, d_in)
    a = gate = up = None
    if act == "swiglu":
        gate, up = ints(d_in, d_ff), ints(d_in, d_ff)
    else:
        a = ints(d_in, d_ff)
    b = ints(d_ff, d_out)
    return MlpInputs(act, "f32", tokens, d_in, d_ff, d_out, seed, x, a, gate, up, b, rng)
