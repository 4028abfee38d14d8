"""The oracle: a plain fp64 CPU implementation of the tensor-parallel MLP.

TEST INFRASTRUCTURE ONLY.  The test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA library in
``tensor_sharded_mlp_b200`` never imports this package and this package never
imports it; the two share only the seeded input generator
(``tensor_sharded_mlp_b200.inputs``), which holds none of the method's
arithmetic.

The arithmetic lives in ``tp_mlp_oracle.c`` (plain C loops, fp64).  This module
compiles it with gcc on first use and marshals numpy arrays into it.

The fused all-reduce + residual add + RMSNorm lives in ``fused_norm_oracle.c``,
the merge of attention partials across KV shards in ``attn_merge_oracle.c``.

Sources (page title and section):
  * "LLM 推理并行化：先找瓶颈，再决定怎么切", §三 2) 张量并行（TP） — the
    tensor_parallel_output function: per rank act(x @ A_i) @ B_i, summed.
  * "大模型推理系统揭秘（07）：Multi-GPU：一张卡不够时如何扩展？", §1.2.2–§1.2.4
    (column/row parallel linears, Z = sum_i Y_i W_2i) and §1.4.3 (SwiGLU).
  * "7.4 推理侧并行", §7.4.2, optimisation 2 — the residual add and RMSNorm
    that follow the all-reduce, fused with it.
  * "LLM 推理并行化：先找瓶颈，再决定怎么切", §三 4) 上下文并行（CP） — decode
    context parallelism: merging the ranks' partial attention results.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = [os.path.join(_HERE, n) for n in ("tp_mlp_oracle.c", "fused_norm_oracle.c", "attn_merge_oracle.c")]
_LIB = os.path.join(_HERE, "libtp_mlp_oracle.so")
_lock = threading.Lock()
_lib = None

ACTS = {"tanh": 0, "swiglu": 1, "identity": 2}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no FMA contraction)."""
    stale = not os.path.exists(_LIB) or any(os.path.getmtime(_LIB) < os.path.getmtime(s) for s in _SRCS)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-o", tmp] + _SRCS + ["-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            fp = ctypes.POINTER(ctypes.c_float)
            dp = ctypes.POINTER(ctypes.c_double)
            fpp = ctypes.POINTER(fp)
            lib.oracle_tp_mlp_sharded.restype = ctypes.c_longlong
            lib.oracle_tp_mlp_sharded.argtypes = [
                fp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, fpp, ctypes.c_int, fpp, dp, dp]
            lib.oracle_tp_mlp_unsharded.restype = ctypes.c_longlong
            lib.oracle_tp_mlp_unsharded.argtypes = [
                fp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                fp, fp, fp, dp]
            lib.oracle_allreduce_residual_rmsnorm.restype = ctypes.c_int
            lib.oracle_allreduce_residual_rmsnorm.argtypes = [
                fp, ctypes.c_int, ctypes.c_int, ctypes.c_int, fp, fp, ctypes.c_double, dp, dp]
            for name in ("oracle_attention_partial", "oracle_merge_attention_partials", "oracle_attention_full"):
                getattr(lib, name).restype = ctypes.c_int
            lib.oracle_attention_partial.argtypes = [fp, fp, fp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                     ctypes.c_double, dp, dp, dp]
            lib.oracle_merge_attention_partials.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, fp, fp, fp, dp]
            lib.oracle_attention_full.argtypes = [fp, fp, fp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_double, dp]
            lib.oracle_max_threads.restype = ctypes.c_int
            lib.oracle_set_threads.argtypes = [ctypes.c_int]
            _lib = lib
    return _lib


def _f32(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != np.float32:
        b = a.astype(np.float32)
        if not np.array_equal(b.astype(a.dtype), a):
            raise ValueError("oracle inputs must hold fp32-representable values")
        a = b
    return np.ascontiguousarray(a)


def _fptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def _act_code(act: str) -> int:
    if act not in ACTS:
        raise ValueError(f"unknown activation {act!r}")
    return ACTS[act]


def tp_mlp_sharded(x, a_shards, b_shards, act: str = "tanh", *, return_partials=False,
                   return_macs=False):
    """Sum over ranks of act(x @ A_i) @ B_i, in fp64.

    x: T x d_in.  tanh/identity: A_i is d_in x f_s; SwiGLU: A_i is d_in x 2 f_s
    laid out [gate_i | up_i].  B_i is f_s x d_out.  The number of A and B
    shards must match (ValueError otherwise), as pairing them strictly does.
    Returns Z (T x d_out, float64); optionally the partials (P x T x d_out) and
    the count of multiply-adds the loops executed.
    """
    a_shards = list(a_shards)
    b_shards = list(b_shards)
    if len(a_shards) != len(b_shards):
        raise ValueError(f"{len(a_shards)} first-projection shards but {len(b_shards)} "
                         "second-projection shards")
    if not a_shards:
        raise ValueError("need at least one rank")
    code = _act_code(act)
    x = _f32(x)
    if x.ndim != 2:
        raise ValueError("x must be 2-D (tokens x d_in)")
    T, d_in = x.shape
    A = [_f32(a) for a in a_shards]
    B = [_f32(b) for b in b_shards]
    P = len(A)
    f_s = B[0].shape[0]
    d_out = B[0].shape[1]
    wa = 2 * f_s if code == ACTS["swiglu"] else f_s
    for a, b in zip(A, B):
        if a.shape != (d_in, wa) or b.shape != (f_s, d_out):
            raise ValueError(f"shard shapes {a.shape}, {b.shape} do not match "
                             f"x {x.shape}, f_s={f_s}, d_out={d_out}, act={act}")
    # NaN-filled: the C code must write every element itself
    z = np.full((T, d_out), np.nan, dtype=np.float64)
    parts = np.full((P, T, d_out), np.nan, dtype=np.float64) if return_partials else None
    fp = ctypes.POINTER(ctypes.c_float)
    arr_a = (fp * P)(*[_fptr(a) for a in A])
    arr_b = (fp * P)(*[_fptr(b) for b in B])
    dp = ctypes.POINTER(ctypes.c_double)
    macs = _load().oracle_tp_mlp_sharded(
        _fptr(x), T, d_in, P * f_s, d_out, code, P, arr_a, P, arr_b,
        z.ctypes.data_as(dp), parts.ctypes.data_as(dp) if parts is not None else None)
    if macs < 0:
        raise ValueError("oracle rejected the arguments")
    out = [z]
    if return_partials:
        out.append(parts)
    if return_macs:
        out.append(int(macs))
    return out[0] if len(out) == 1 else tuple(out)


def tp_mlp_partials(x, a_shards, b_shards, act: str = "tanh"):
    """Every rank's partial Z_i = act(x @ A_i) @ B_i (P x T x d_out, fp64)."""
    return tp_mlp_sharded(x, a_shards, b_shards, act, return_partials=True)[1]


def tp_mlp_unsharded(x, a, b, act: str = "tanh", a_up=None, *, return_macs=False):
    """act(x @ A) @ B on the full matrices, in fp64 (SwiGLU: a = gate, a_up = up)."""
    code = _act_code(act)
    if (code == ACTS["swiglu"]) != (a_up is not None):
        raise ValueError("SwiGLU needs both gate (a) and up (a_up); other activations take one")
    x = _f32(x)
    a = _f32(a)
    b = _f32(b)
    T, d_in = x.shape
    d_ff = a.shape[1]
    d_out = b.shape[1]
    if a.shape != (d_in, d_ff) or b.shape != (d_ff, d_out):
        raise ValueError("shape mismatch")
    up = None
    if a_up is not None:
        up = _f32(a_up)
        if up.shape != a.shape:
            raise ValueError("gate and up shapes differ")
    z = np.full((T, d_out), np.nan, dtype=np.float64)
    macs = _load().oracle_tp_mlp_unsharded(
        _fptr(x), T, d_in, d_ff, d_out, code, _fptr(a), _fptr(up) if up is not None else None,
        _fptr(b), z.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if macs < 0:
        raise ValueError("oracle rejected the arguments")
    return (z, int(macs)) if return_macs else z


def allreduce_residual_rmsnorm(partials, residual, gamma, eps: float):
    """The rank sum followed by the residual add and RMSNorm, in fp64.

    partials: P x T x d (every rank's Z_i); residual: T x d; gamma: d.
    h = residual + sum_i Z_i (ranks in order); y = h / sqrt(mean(h^2) + eps) * gamma,
    row by row.  Returns (y, h), both T x d float64.
    """
    p = _f32(partials)
    r = _f32(residual)
    g = _f32(gamma)
    if p.ndim != 3 or r.ndim != 2 or g.ndim != 1:
        raise ValueError("partials must be P x T x d, residual T x d, gamma d")
    P, T, d = p.shape
    if r.shape != (T, d) or g.shape != (d,):
        raise ValueError(f"residual {r.shape} / gamma {g.shape} do not match partials {p.shape}")
    y = np.full((T, d), np.nan, dtype=np.float64)
    h = np.full((T, d), np.nan, dtype=np.float64)
    dp = ctypes.POINTER(ctypes.c_double)
    rc = _load().oracle_allreduce_residual_rmsnorm(_fptr(p), P, T, d, _fptr(r), _fptr(g), float(eps),
                                                   y.ctypes.data_as(dp), h.ctypes.data_as(dp))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return y, h


def attention_partial(q, k, v, scale: float):
    """One rank's partial attention over its KV shard, in fp64: per query row the
    maximum score, the sum of exp(score - maximum) and the exp-weighted sum of
    the values.  q: rows x D, k and v: n_keys x D (n_keys may be 0)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    rows, D = q.shape
    n = k.shape[0]
    if k.shape != (n, D) or v.shape != (n, D):
        raise ValueError("k and v must be n_keys x D")
    m = np.full(rows, np.nan)
    s = np.full(rows, np.nan)
    w = np.full((rows, D), np.nan)
    dp = ctypes.POINTER(ctypes.c_double)
    if _load().oracle_attention_partial(_fptr(q), _fptr(k), _fptr(v), rows, n, D, float(scale),
                                        m.ctypes.data_as(dp), s.ctypes.data_as(dp), w.ctypes.data_as(dp)) != 0:
        raise ValueError("oracle rejected the arguments")
    return m, s, w


def merge_attention_partials(maximum, exp_sum, weighted):
    """Merge P ranks' partials (maximum, exp_sum: P x rows; weighted: P x rows x D),
    in fp64: rescale each rank by exp(its maximum - the global maximum), add,
    divide.  Rows with every rank empty (maximum -inf) merge to zeros."""
    m, s, w = _f32(maximum), _f32(exp_sum), _f32(weighted)
    if m.ndim != 2 or s.shape != m.shape or w.ndim != 3 or w.shape[:2] != m.shape:
        raise ValueError("maximum and exp_sum must be P x rows, weighted P x rows x D")
    P, rows, D = w.shape
    out = np.full((rows, D), np.nan)
    if _load().oracle_merge_attention_partials(P, rows, D, _fptr(m), _fptr(s), _fptr(w),
                                               out.ctypes.data_as(ctypes.POINTER(ctypes.c_double))) != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def attention_full(q, k, v, scale: float):
    """Softmax attention of every query row over all keys, in fp64."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    rows, D = q.shape
    out = np.full((rows, D), np.nan)
    if _load().oracle_attention_full(_fptr(q), _fptr(k), _fptr(v), rows, k.shape[0], D, float(scale),
                                     out.ctypes.data_as(ctypes.POINTER(ctypes.c_double))) != 0:
        raise ValueError("oracle rejected the arguments")
    return out
