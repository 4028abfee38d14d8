"""Analytic work counts for the tensor-parallel MLP (host logic, no GPU).

Sources:
  * "7.4 推理侧并行", §7.4.1, per-token FLOPs table: a forward pass costs 2N
    FLOPs per token for N parameters (one multiply and one add each); decode at
    batch 1 reads every weight once (140 GB of FP16 for 70B parameters).
  * "7.4 推理侧并行", §7.4.2: one tensor-parallel all-reduce carries
    B * S * d_model * bytes.

"Algorithmic" bytes are what the method must move through HBM in one forward:
every weight once, X once, the output once, and the intermediate activation H
written once and read once.  Elementwise activation work is not counted as
FLOPs.
"""
from __future__ import annotations

import hashlib
import os
import re

ELEM_BYTES = {"f32": 4, "bf16": 2}


def mlp_params(d_in: int, d_ff: int, d_out: int, act: str) -> int:
    """Weight count N: first projection(s) plus the second projection."""
    first = 2 * d_in * d_ff if act == "swiglu" else d_in * d_ff
    return first + d_ff * d_out


def forward_flops(tokens: int, d_in: int, d_ff: int, d_out: int, act: str) -> int:
    """2 N FLOPs per token."""
    return 2 * mlp_params(d_in, d_ff, d_out, act) * tokens


def weight_bytes(d_in: int, d_ff: int, d_out: int, act: str, dtype: str) -> int:
    return mlp_params(d_in, d_ff, d_out, act) * ELEM_BYTES[dtype]


def algorithmic_bytes(tokens: int, d_in: int, d_ff: int, d_out: int, act: str,
                      dtype: str) -> int:
    """Weights once + X once + output once + H written and read once."""
    e = ELEM_BYTES[dtype]
    return (weight_bytes(d_in, d_ff, d_out, act, dtype)
            + tokens * d_in * e + tokens * d_out * e + 2 * tokens * d_ff * e)


def gemm1_bytes(tokens, d_in, d_ff, act, dtype) -> int:
    """First projection + activation: its weights, X, and H written."""
    e = ELEM_BYTES[dtype]
    w = (2 if act == "swiglu" else 1) * d_in * d_ff * e
    return w + tokens * d_in * e + tokens * d_ff * e


def gemm2_bytes(tokens, d_ff, d_out, dtype) -> int:
    """Second projection + shard sum: its weights, H read, output written."""
    e = ELEM_BYTES[dtype]
    return d_ff * d_out * e + tokens * d_ff * e + tokens * d_out * e


def gemm1_flops(tokens, d_in, d_ff, act) -> int:
    return 2 * tokens * d_in * d_ff * (2 if act == "swiglu" else 1)


def gemm2_flops(tokens, d_ff, d_out) -> int:
    return 2 * tokens * d_ff * d_out


def columns_per_rank(columns: int, tp: int) -> int:
    """A column split gives each of the tp ranks columns / tp columns (even splits only)."""
    if tp < 1 or columns % tp:
        raise ValueError(f"{columns} columns do not split evenly over {tp} ranks")
    return columns // tp


def allreduce_bytes(batch: int, seq: int, d_model: int, elem_bytes: int) -> int:
    """Bytes one tensor-parallel all-reduce carries: B * S * d_model * bytes."""
    return batch * seq * d_model * elem_bytes


def fused_norm_bytes(tp: int, tokens: int, d_model: int, dtype: str) -> int:
    """Bytes the fused all-reduce + residual add + RMSNorm must move: every
    rank's fp32 partial row read once, the residual and gamma read, y and the
    updated residual written ("7.4 推理侧并行" §7.4.2, optimisation 2)."""
    e = 4 if dtype == "f32" else 2
    n = tokens * d_model
    return tp * n * 4 + n * e + d_model * e + 2 * n * e


def unfused_norm_bytes(tp: int, tokens: int, d_model: int, dtype: str) -> int:
    """The same step as three kernels (all-reduce writing Z in the activation
    dtype, residual add, RMSNorm): Z and h each make one extra round trip."""
    e = 4 if dtype == "f32" else 2
    n = tokens * d_model
    return fused_norm_bytes(tp, tokens, d_model, dtype) + 2 * (2 * n * e)


# Source files that define each kernel family (for "was this profile taken on
# the current kernel?" checks).
_KERNEL_SOURCES = {
    "fused_norm": ["fused_norm.cu", "vec_io.cuh", "common.cuh", "tc_ptx.cuh"],
    "attn_merge": ["attn_merge.cu", "vec_io.cuh", "common.cuh"],
    "gemv": ["gemv.cu", "common.cuh", "streamk.cuh", "tc_ptx.cuh"],
    "tc_skinny": ["tc_gemm.cu", "common.cuh", "streamk.cuh", "tc_ptx.cuh"],
    "tc_wide": ["tc_gemm.cu", "common.cuh", "streamk.cuh", "tc_ptx.cuh"],
    "tc_wide256": ["tc_gemm.cu", "common.cuh", "streamk.cuh", "tc_ptx.cuh"],
    "tc_pair": ["tc_gemm.cu", "common.cuh", "streamk.cuh", "tc_ptx.cuh"],
    "tc_pair2": ["tc_gemm.cu", "common.cuh", "streamk.cuh", "tc_ptx.cuh"],
    "tc_fused": ["tc_gemm.cu", "common.cuh", "streamk.cuh", "tc_ptx.cuh"],
    "simt": ["simt.cu", "common.cuh"],
}


def _code_only(text: str) -> str:
    """C/CUDA source without comments or layout: what the compiler sees of it."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(plan: str) -> str:
    """Hash of the code (comments and whitespace ignored) of a kernel family's sources."""
    d = os.path.join(os.path.dirname(os.path.abspath(__file__)), "csrc")
    h = hashlib.sha256()
    for n in _KERNEL_SOURCES.get(plan, sorted(os.listdir(d))):
        with open(os.path.join(d, n), encoding="utf-8") as f:
            h.update(n.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]
