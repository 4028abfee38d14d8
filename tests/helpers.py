"""Shared helpers for the GPU tests: uploads and the tolerance rule.

Tolerance: max |gpu - ref| <= k * max |ref| over every checked element, with
k = 1e-5 for fp32 inputs and k = 2e-2 for bf16 inputs (fp32 accumulation),
the bounds the workload definitions state.
"""
import numpy as np
import torch

TOL = {"f32": 1e-5, "bf16": 2e-2}
TORCH = {"f32": torch.float32, "bf16": torch.bfloat16}


def dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    """fp32 array holding dtype-representable values -> CUDA tensor of that dtype (exact)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    return t.to(TORCH[dtype]).contiguous()


def rel_err(got, ref) -> float:
    got = got.float().cpu().numpy().astype(np.float64) if isinstance(got, torch.Tensor) else got
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.max(np.abs(ref))
    err = np.max(np.abs(got - ref))
    return float(err / scale) if scale > 0 else float(err)


def assert_close(got, ref, dtype: str, what: str = ""):
    r = rel_err(got, ref)
    assert r <= TOL[dtype], f"{what}: max|err|/max|ref| = {r:.3e} > {TOL[dtype]:.0e}"
    return r
