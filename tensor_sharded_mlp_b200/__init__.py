"""tensor_sharded_mlp_b200 — the tensor-parallel two-projection MLP on one B200.

For each tensor-parallel rank i: H_i = act(X A_i) (column-sharded first
projection, act = tanh or SwiGLU), Z_i = H_i B_i (row-sharded second
projection), Z = sum_i Z_i.  All shards live in one GPU's HBM, so the
all-reduce is an on-device sum fused into the second projection.

The compute runs in the CUDA library ``libtp_mlp.so`` (C ABI declared in
``include/tp_mlp.h``); ``tensor_sharded_mlp_b200.binding`` marshals torch
tensors into it.  The library is loaded on first use and a missing library is
an error: there is no CPU fallback.
"""
__all__ = ["binding", "inputs", "counts"]


def __getattr__(name):
    if name == "binding":
        import importlib
        return importlib.import_module(".binding", __name__)
    raise AttributeError(name)
