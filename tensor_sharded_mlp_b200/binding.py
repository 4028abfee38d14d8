"""Thin Python binding of ``libtp_mlp.so`` (argument marshalling only).

The functions carry the C ABI's names (``include/tp_mlp.h``) and take torch
tensors where the C call takes device pointers; every step of the MLP runs in
the library's CUDA kernels.  Tensors supply device memory and
``torch.cuda.current_stream()`` (or an explicit stream) supplies the stream.

If the library is missing this module raises on import: there is no fallback.
``TpMlp`` is a small convenience wrapper that owns the handle and a
torch-allocated workspace.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtp_mlp.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"CUDA library not built: {_LIB_PATH} is missing "
                      "(run python -m tensor_sharded_mlp_b200.build)")
_lib = ctypes.CDLL(_LIB_PATH)

ACT = {"tanh": 0, "swiglu": 1, "identity": 2}
DTYPE = {"f32": 0, "bf16": 1}
TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}
PLAN = {"auto": 0, "simt": 1, "gemv": 2, "tc": 3, "tc_wide": 4, "tc_skinny": 5, "tc_wide256": 6, "tc_pair": 7,
        "tc_pair2": 8, "tc_fused": 9}
PLAN_NAME = {v: k for k, v in PLAN.items()}
STATUS = {0: "OK", 1: "ERR_INVALID_ARG", 2: "ERR_SHAPE", 3: "ERR_ALIGNMENT", 4: "ERR_UNSUPPORTED",
          5: "ERR_CUDA", 6: "ERR_TIMEOUT", 7: "ERR_WORKSPACE"}

_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t
_vpp = ctypes.POINTER(ctypes.c_void_p)

_SIGS = {
    "tp_mlp_create": (_i, [ctypes.POINTER(_vp), _i, _i, _i, _i, _i, _i, _i]),
    "tp_mlp_destroy": (_i, [_vp]),
    "tp_mlp_workspace_bytes": (_sz, [_vp, _i]),
    "tp_mlp_set_workspace": (_i, [_vp, _vp, _sz]),
    "tp_mlp_forward": (_i, [_vp, _vp, _i, _vpp, _vpp, _i, _i, _vp, _vp]),
    "tp_mlp_partials": (_i, [_vp, _vp, _i, _vpp, _vpp, _i, _i, _vp, _vp]),
    "tp_mlp_packed_bytes": (_sz, [_vp]),
    "tp_mlp_pack": (_i, [_vp, _vpp, _vpp, _vp, _vp]),
    "tp_mlp_unpack": (_i, [_vp, _vp, _vpp, _vpp, _vp]),
    "tp_mlp_forward_packed": (_i, [_vp, _vp, _i, _vp, _vp, _vp]),
    "tp_mlp_set_plan": (_i, [_vp, _i]),
    "tp_mlp_set_splitk": (_i, [_vp, _i]),
    "tp_mlp_allreduce_residual_rmsnorm": (_i, [_vp, _i, _i, _i, _vp, _vp, ctypes.c_float, _i, _vp, _vp, _vp]),
    "tp_mlp_merge_attention_partials": (_i, [_i, _i, _i, _vp, _vp, _vp, _i, _vp, _vp]),
    "tp_mlp_set_profile_events": (_i, [_vp, _vpp, _i]),
    "tp_mlp_get_device_status": (_i, [_vp]),
    "tp_mlp_selftest_bounded_wait": (_i, [_vp, ctypes.c_uint, _vp]),
    "tp_mlp_last_plan": (_i, [_vp]),
    "tp_mlp_last_launches": (_i, [_vp]),
    "tp_mlp_status_string": (ctypes.c_char_p, [_i]),
    "tp_mlp_decode_forward_static": (_i, [_i, _i, _i, _i, _i, _vp, _i, _vp, _vp, _vp]),
    "tp_mlp_decode_static_status": (_i, []),
    "tp_mlp_xgpu_comm_bytes": (_sz, [_vp]),
    "tp_mlp_xgpu_forward": (_i, [_vp, _i, _i, _vp, _i, _vpp, _vpp, _vpp, _vpp, _vp]),
    "tp_mlp_xgpu_sp_forward": (_i, [_vp, _i, _i, _vpp, _i, _vpp, _vpp, _vpp, _vpp, _vp]),
    "tp_mlp_ipc_get_handle": (_i, [_vp, _vp, ctypes.POINTER(_sz)]),
    "tp_mlp_ipc_open_handle": (_i, [_vp, _sz, ctypes.POINTER(_vp)]),
    "tp_mlp_ipc_close_handle": (_i, [_vp, _sz]),
    "tp_mlp_copy_async": (_i, [_vp, _vp, _sz, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)


class TpMlpError(RuntimeError):
    def __init__(self, call: str, status: int):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{call} failed: {self.name} "
                         f"({_lib.tp_mlp_status_string(status).decode()})")


def _check(call: str, status: int) -> None:
    if status != 0:
        raise TpMlpError(call, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr_array(ts: Sequence[torch.Tensor], n: int):
    # the C call reads exactly n pointers from this array
    if len(ts) != n:
        raise ValueError(f"{len(ts)} shards given for tp_degree={n}")
    for t in ts:
        if not t.is_contiguous():
            raise ValueError("shards must be contiguous")
    arr = (ctypes.c_void_p * max(1, len(ts)))(*[t.data_ptr() for t in ts])
    return ctypes.cast(arr, _vpp), arr


# --- functions with the C ABI's names ------------------------------------------

def tp_mlp_create(d_model: int, d_ff: int, d_out: int, tp_degree: int, act: str, dtype: str,
                  max_tokens: int) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check("tp_mlp_create", _lib.tp_mlp_create(ctypes.byref(h), d_model, d_ff, d_out, tp_degree,
                                               ACT[act], DTYPE[dtype], max_tokens))
    return h


def tp_mlp_destroy(h) -> None:
    _check("tp_mlp_destroy", _lib.tp_mlp_destroy(h))


def tp_mlp_workspace_bytes(h, tokens: int) -> int:
    return int(_lib.tp_mlp_workspace_bytes(h, tokens))


def tp_mlp_set_workspace(h, ws: Optional[torch.Tensor]) -> None:
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("tp_mlp_set_workspace", _lib.tp_mlp_set_workspace(h, _ptr(ws), nbytes))


def tp_mlp_forward(h, x: torch.Tensor, A_shards, B_shards, tp_degree: int, act: str,
                   out: torch.Tensor, stream=None) -> None:
    a, _ka = _ptr_array(A_shards, tp_degree)
    b, _kb = _ptr_array(B_shards, tp_degree)
    _check("tp_mlp_forward", _lib.tp_mlp_forward(h, _ptr(x), x.shape[0], a, b, tp_degree, ACT[act],
                                                 _ptr(out), _stream(stream)))


def tp_mlp_partials(h, x: torch.Tensor, A_shards, B_shards, tp_degree: int, act: str,
                    partials: torch.Tensor, stream=None) -> None:
    a, _ka = _ptr_array(A_shards, tp_degree)
    b, _kb = _ptr_array(B_shards, tp_degree)
    _check("tp_mlp_partials", _lib.tp_mlp_partials(h, _ptr(x), x.shape[0], a, b, tp_degree,
                                                   ACT[act], _ptr(partials), _stream(stream)))


def tp_mlp_packed_bytes(h) -> int:
    return int(_lib.tp_mlp_packed_bytes(h))


def tp_mlp_pack(h, A_shards, B_shards, packed: torch.Tensor, tp_degree: int, stream=None) -> None:
    a, _ka = _ptr_array(A_shards, tp_degree)
    b, _kb = _ptr_array(B_shards, tp_degree)
    _check("tp_mlp_pack", _lib.tp_mlp_pack(h, a, b, _ptr(packed), _stream(stream)))


def tp_mlp_unpack(h, packed: torch.Tensor, A_shards, B_shards, tp_degree: int, stream=None) -> None:
    a, _ka = _ptr_array(A_shards, tp_degree)
    b, _kb = _ptr_array(B_shards, tp_degree)
    _check("tp_mlp_unpack", _lib.tp_mlp_unpack(h, _ptr(packed), a, b, _stream(stream)))


def tp_mlp_forward_packed(h, x: torch.Tensor, packed: torch.Tensor, out: torch.Tensor,
                          stream=None) -> None:
    _check("tp_mlp_forward_packed", _lib.tp_mlp_forward_packed(h, _ptr(x), x.shape[0], _ptr(packed),
                                                               _ptr(out), _stream(stream)))


def tp_mlp_set_plan(h, plan: str) -> None:
    _check("tp_mlp_set_plan", _lib.tp_mlp_set_plan(h, PLAN[plan]))


SPLITK = {"auto": 0, "in_kernel": 1, "separate": 2, "cluster": 3}


def tp_mlp_set_splitk(h, mode: str) -> None:
    _check("tp_mlp_set_splitk", _lib.tp_mlp_set_splitk(h, SPLITK[mode]))


def tp_mlp_set_profile_events(h, events) -> None:
    """events: torch.cuda.Event objects (timing enabled, already recorded once so
    that they exist), or None to turn the hook off."""
    if not events:
        _check("tp_mlp_set_profile_events", _lib.tp_mlp_set_profile_events(h, None, 0))
        return
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _check("tp_mlp_set_profile_events",
           _lib.tp_mlp_set_profile_events(h, ctypes.cast(arr, _vpp), len(events)))


def tp_mlp_get_device_status(h) -> None:
    _check("tp_mlp_get_device_status", _lib.tp_mlp_get_device_status(h))


def tp_mlp_selftest_bounded_wait(h, wait_us: int, stream=None) -> None:
    _check("tp_mlp_selftest_bounded_wait", _lib.tp_mlp_selftest_bounded_wait(h, wait_us, _stream(stream)))


def tp_mlp_last_plan(h) -> str:
    return PLAN_NAME.get(_lib.tp_mlp_last_plan(h), "none")


def tp_mlp_last_launches(h) -> int:
    return int(_lib.tp_mlp_last_launches(h))


def tp_mlp_status_string(status: int) -> str:
    return _lib.tp_mlp_status_string(status).decode()


def tp_mlp_decode_forward_static(d_model: int, d_ff: int, d_out: int, tp_degree: int, act: str,
                                 x: torch.Tensor, packed: torch.Tensor, out: torch.Tensor,
                                 stream=None) -> None:
    """Decode forward for callers that cannot allocate device memory: its
    scratch is a fixed array inside the library, so no workspace is passed.
    x (T, d_model) and out (T, d_out): contiguous CUDA bfloat16; packed: the
    contiguous CUDA buffer tp_mlp_pack wrote for this shape."""
    for t, what in ((x, "x"), (out, "out")):
        if t.dtype != torch.bfloat16 or t.dim() != 2 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{what} must be a contiguous 2-D CUDA bfloat16 tensor")
    if x.shape[1] != d_model or out.shape != (x.shape[0], d_out):
        raise ValueError(f"x must be (T, {d_model}) and out (T, {d_out}); got {tuple(x.shape)}, {tuple(out.shape)}")
    if not packed.is_cuda or not packed.is_contiguous():
        raise ValueError("packed must be a contiguous CUDA tensor")
    _check("tp_mlp_decode_forward_static",
           _lib.tp_mlp_decode_forward_static(d_model, d_ff, d_out, tp_degree, ACT[act], _ptr(x), x.shape[0],
                                             _ptr(packed), _ptr(out), _stream(stream)))


def tp_mlp_decode_static_status() -> None:
    """Raise TpMlpError(ERR_TIMEOUT) if a kernel of an earlier
    tp_mlp_decode_forward_static call on the current device gave up a bounded
    wait (and clear that record); synchronises the device."""
    _check("tp_mlp_decode_static_status", _lib.tp_mlp_decode_static_status())


def tp_mlp_xgpu_comm_bytes(h) -> int:
    return int(_lib.tp_mlp_xgpu_comm_bytes(h))


def _raw_ptr_array(ptrs: Sequence[int]):
    arr = (ctypes.c_void_p * max(1, len(ptrs)))(*[int(p) for p in ptrs])
    return ctypes.cast(arr, _vpp), arr


def tp_mlp_xgpu_forward(h, rank0: int, x: torch.Tensor, A_local, B_local, comm_ptrs: Sequence[int],
                        outs, stream=None) -> None:
    """Ranks rank0 .. rank0 + len(A_local) - 1 of a tensor-parallel MLP whose
    all-reduce crosses GPUs (one-shot, fused into the second projection).
    comm_ptrs: every rank's exchange buffer address as seen by this process."""
    n = len(A_local)
    if len(B_local) != n or len(outs) != n:
        raise ValueError("A_local, B_local and outs need one entry per local rank")
    for t in list(A_local) + list(B_local) + list(outs) + [x]:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("x, shards and outputs must be contiguous CUDA bfloat16 tensors")
    a, _ka = _ptr_array(A_local, n)
    b, _kb = _ptr_array(B_local, n)
    o, _ko = _ptr_array(outs, n)
    c, _kc = _raw_ptr_array(comm_ptrs)
    _check("tp_mlp_xgpu_forward", _lib.tp_mlp_xgpu_forward(h, rank0, n, _ptr(x), x.shape[0], a, b, c, o,
                                                           _stream(stream)))


def tp_mlp_xgpu_sp_forward(h, rank0: int, x_local, A_local, B_local, comm_ptrs: Sequence[int], outs,
                           stream=None) -> None:
    """Sequence-parallel form: x_local[i] holds local rank i's tokens / tp rows;
    the rows are gathered before the first projection and the second
    projection's exchange is a reduce-scatter (outs[i]: rank i's own rows)."""
    n = len(A_local)
    if len(B_local) != n or len(outs) != n or len(x_local) != n:
        raise ValueError("x_local, A_local, B_local and outs need one entry per local rank")
    for t in list(x_local) + list(A_local) + list(B_local) + list(outs):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("rows, shards and outputs must be contiguous CUDA bfloat16 tensors")
    tp = len(comm_ptrs)
    tokens = x_local[0].shape[0] * tp
    xs, _kx = _ptr_array(x_local, n)
    a, _ka = _ptr_array(A_local, n)
    b, _kb = _ptr_array(B_local, n)
    o, _ko = _ptr_array(outs, n)
    c, _kc = _raw_ptr_array(comm_ptrs)
    _check("tp_mlp_xgpu_sp_forward", _lib.tp_mlp_xgpu_sp_forward(h, rank0, n, xs, tokens, a, b, c, o,
                                                                 _stream(stream)))


def tp_mlp_ipc_get_handle(t: torch.Tensor):
    """(64-byte handle, offset) of the device allocation holding tensor t."""
    buf = ctypes.create_string_buffer(64)
    off = ctypes.c_size_t()
    _check("tp_mlp_ipc_get_handle", _lib.tp_mlp_ipc_get_handle(_ptr(t), buf, ctypes.byref(off)))
    return bytes(buf.raw), int(off.value)


def tp_mlp_ipc_open_handle(handle: bytes, offset: int) -> int:
    """Map another process's allocation; returns the device address of handle + offset."""
    if len(handle) != 64:
        raise ValueError("an IPC handle is 64 bytes")
    buf = ctypes.create_string_buffer(handle, 64)
    p = ctypes.c_void_p()
    _check("tp_mlp_ipc_open_handle", _lib.tp_mlp_ipc_open_handle(buf, offset, ctypes.byref(p)))
    return int(p.value)


def tp_mlp_ipc_close_handle(ptr: int, offset: int) -> None:
    _check("tp_mlp_ipc_close_handle", _lib.tp_mlp_ipc_close_handle(ctypes.c_void_p(ptr), offset))


def tp_mlp_allreduce_residual_rmsnorm(partials: torch.Tensor, residual: torch.Tensor, gamma: torch.Tensor,
                                      eps: float, y: Optional[torch.Tensor] = None,
                                      residual_out: Optional[torch.Tensor] = None, stream=None):
    """The rank sum of fp32 partials (P x T x d) fused with the residual add and
    RMSNorm: h = residual + sum_i partials[i], y = h / sqrt(mean(h^2) + eps) * gamma.
    residual_out may be residual itself (in-place update).  Returns (y, residual_out)."""
    if partials.dtype != torch.float32 or partials.dim() != 3 or not partials.is_contiguous():
        raise ValueError("partials must be a contiguous float32 tensor (P, T, d)")
    P, T, d = partials.shape
    dt = residual.dtype
    if dt not in (torch.float32, torch.bfloat16):
        raise ValueError("residual must be float32 or bfloat16")
    if residual.shape != (T, d) or gamma.shape != (d,) or gamma.dtype != dt:
        raise ValueError("residual must be (T, d) and gamma (d,), of one dtype")
    for t in (partials, residual, gamma):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    if y is None:
        y = torch.empty_like(residual)
    if residual_out is None:
        residual_out = torch.empty_like(residual)
    for t in (y, residual_out):
        if t.shape != (T, d) or t.dtype != dt or not t.is_contiguous():
            raise ValueError("y / residual_out must be contiguous (T, d) tensors of the residual's dtype")
    _check("tp_mlp_allreduce_residual_rmsnorm",
           _lib.tp_mlp_allreduce_residual_rmsnorm(_ptr(partials), P, T, d, _ptr(residual), _ptr(gamma),
                                                  float(eps), DTYPE["f32" if dt == torch.float32 else "bf16"],
                                                  _ptr(y), _ptr(residual_out), _stream(stream)))
    return y, residual_out


def tp_mlp_merge_attention_partials(maximum: torch.Tensor, exp_sum: torch.Tensor, weighted: torch.Tensor,
                                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Merge P ranks' partial attention results: maximum, exp_sum (P, rows) float32,
    weighted (P, rows, head_dim) float32 or bfloat16 -> out (rows, head_dim)."""
    if weighted.dim() != 3 or weighted.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("weighted must be a float32 or bfloat16 tensor (P, rows, head_dim)")
    P, rows, D = weighted.shape
    for t in (maximum, exp_sum):
        if t.dtype != torch.float32 or t.shape != (P, rows):
            raise ValueError("maximum and exp_sum must be float32 (P, rows)")
    for t in (maximum, exp_sum, weighted):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty(rows, D, dtype=weighted.dtype, device=weighted.device)
    if out.shape != (rows, D) or out.dtype != weighted.dtype or not out.is_contiguous():
        raise ValueError("out must be a contiguous (rows, head_dim) tensor of weighted's dtype")
    _check("tp_mlp_merge_attention_partials",
           _lib.tp_mlp_merge_attention_partials(P, rows, D, _ptr(maximum), _ptr(exp_sum), _ptr(weighted),
                                                DTYPE["f32" if weighted.dtype == torch.float32 else "bf16"],
                                                _ptr(out), _stream(stream)))
    return out


def tp_mlp_copy_async(dst: torch.Tensor, src: torch.Tensor, stream=None) -> torch.Tensor:
    """Copy src's bytes into dst on the stream.  Each may be a CUDA tensor of the
    current device or a pinned host tensor; both contiguous, the same size in
    bytes, not overlapping.  Decode-sized copies run as a library kernel."""
    n = src.numel() * src.element_size()
    if not src.is_contiguous() or not dst.is_contiguous() or dst.numel() * dst.element_size() != n:
        raise ValueError("src and dst must be contiguous tensors of the same size in bytes")
    for t in (src, dst):
        if not t.is_cuda and not t.is_pinned():
            raise ValueError("host tensors must be pinned (page-locked)")
    _check("tp_mlp_copy_async", _lib.tp_mlp_copy_async(_ptr(dst), _ptr(src), n, _stream(stream)))
    return dst


# --- convenience wrapper -----------------------------------------------------------

class TpMlp:
    """One MLP shape: handle + workspace.  Tensors must live on the current CUDA device."""

    def __init__(self, d_model: int, d_ff: int, tp: int, act: str = "tanh", dtype: str = "bf16",
                 max_tokens: int = 32, d_out: Optional[int] = None, device=None):
        self.d_model, self.d_ff, self.tp, self.act, self.dtype = d_model, d_ff, tp, act, dtype
        self.d_out = d_model if d_out is None else d_out
        self.max_tokens = max_tokens
        self.device = torch.device("cuda" if device is None else device)
        self.h = tp_mlp_create(d_model, d_ff, self.d_out, tp, act, dtype, max_tokens)
        nbytes = tp_mlp_workspace_bytes(self.h, max_tokens)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        tp_mlp_set_workspace(self.h, self.workspace)

    def __del__(self):
        h = getattr(self, "h", None)
        if h is not None and _lib is not None:   # module globals are gone at interpreter exit
            _lib.tp_mlp_destroy(h)
            self.h = None

    @property
    def torch_dtype(self):
        return TORCH_DTYPE[self.dtype]

    def _out(self, x, out):
        if out is None:
            out = torch.empty(x.shape[0], self.d_out, dtype=self.torch_dtype, device=x.device)
        return out

    def _check_x(self, x):
        if x.dtype != self.torch_dtype or x.dim() != 2 or x.shape[1] != self.d_model or \
                not x.is_contiguous() or not x.is_cuda:
            raise ValueError(f"x must be a contiguous CUDA {self.torch_dtype} tensor (T, {self.d_model})")

    def _check_shards(self, A_shards, B_shards):
        if len(A_shards) != len(B_shards):
            raise ValueError(f"{len(A_shards)} first-projection shards but {len(B_shards)} "
                             "second-projection shards")
        for t in list(A_shards) + list(B_shards):
            if t.dtype != self.torch_dtype or not t.is_cuda:
                raise ValueError(f"shards must be CUDA {self.torch_dtype} tensors")

    def forward(self, x, A_shards, B_shards, out=None, stream=None):
        self._check_x(x)
        self._check_shards(A_shards, B_shards)
        out = self._out(x, out)
        tp_mlp_forward(self.h, x, A_shards, B_shards, len(A_shards), self.act, out, stream)
        return out

    def partials(self, x, A_shards, B_shards, out=None, stream=None):
        if out is None:
            out = torch.empty(self.tp, x.shape[0], self.d_out, dtype=torch.float32, device=x.device)
        self._check_x(x)
        self._check_shards(A_shards, B_shards)
        tp_mlp_partials(self.h, x, A_shards, B_shards, len(A_shards), self.act, out, stream)
        return out

    def pack(self, A_shards, B_shards, stream=None):
        self._check_shards(A_shards, B_shards)
        packed = torch.empty(tp_mlp_packed_bytes(self.h), dtype=torch.uint8, device=self.device)
        tp_mlp_pack(self.h, A_shards, B_shards, packed, self.tp, stream)
        return packed

    def unpack(self, packed, stream=None):
        fs = self.d_ff // self.tp
        wa = 2 * fs if self.act == "swiglu" else fs
        A = [torch.empty(self.d_model, wa, dtype=self.torch_dtype, device=self.device)
             for _ in range(self.tp)]
        B = [torch.empty(fs, self.d_out, dtype=self.torch_dtype, device=self.device)
             for _ in range(self.tp)]
        tp_mlp_unpack(self.h, packed, A, B, self.tp, stream)
        return A, B

    def forward_packed(self, x, packed, out=None, stream=None):
        self._check_x(x)
        out = self._out(x, out)
        tp_mlp_forward_packed(self.h, x, packed, out, stream)
        return out

    def set_plan(self, plan: str):
        tp_mlp_set_plan(self.h, plan)

    def set_splitk(self, mode: str):
        tp_mlp_set_splitk(self.h, mode)

    @property
    def last_plan(self) -> str:
        return tp_mlp_last_plan(self.h)

    @property
    def last_launches(self) -> int:
        return tp_mlp_last_launches(self.h)


class GraphStep:
    """A whole decode/prefill step replayed as one CUDA graph.

    Per call: copy the step's input from a pinned host buffer to the device,
    run tp_mlp_forward_packed, copy the result back to a pinned host buffer
    (both copies by tp_mlp_copy_async: a kernel at decode sizes), and wait for
    it.  Capturing these into a graph once removes the per-kernel launch cost
    from every later step (the pages put it at 5-10 us per kernel in a decode
    step, "7.4 推理侧并行" §7.4.2).  The library's calls allocate
    nothing and take no host-side decisions that change between replays, so
    they are safe to capture; the handle's workspace and the packed weights
    must outlive the step.

        step = GraphStep(mlp, packed, tokens)
        step.x_host.copy_(x)          # or step(x) to copy and run
        out = step()                  # pinned host tensor, valid until the next call

    A call replays the graph on the caller's current CUDA stream and waits for it.
    """

    def __init__(self, mlp: "TpMlp", packed: torch.Tensor, tokens: int):
        dt = mlp.torch_dtype
        self.mlp, self.packed = mlp, packed
        self.x_host = torch.zeros(tokens, mlp.d_model, dtype=dt).pin_memory()
        self.out_host = torch.zeros(tokens, mlp.d_out, dtype=dt).pin_memory()
        self.x_dev = torch.zeros(tokens, mlp.d_model, dtype=dt, device=mlp.device)
        self.out_dev = torch.empty(tokens, mlp.d_out, dtype=dt, device=mlp.device)
        self.stream = torch.cuda.Stream(device=mlp.device)
        self.stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(self.stream):          # warm-up outside capture
            self._body()
        self.stream.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=self.stream):
            self._body()
        self.launches = mlp.last_launches

    def _body(self):
        tp_mlp_copy_async(self.x_dev, self.x_host)
        self.mlp.forward_packed(self.x_dev, self.packed, out=self.out_dev)
        tp_mlp_copy_async(self.out_host, self.out_dev)

    def __call__(self, x: Optional[torch.Tensor] = None) -> torch.Tensor:
        if x is not None:
            self.x_host.copy_(x)
        stream = torch.cuda.current_stream(self.mlp.device)
        self.graph.replay()      # on the caller's current stream, after its earlier work
        stream.synchronize()
        return self.out_host
