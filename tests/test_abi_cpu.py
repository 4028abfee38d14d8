"""C ABI checks that need no GPU: exports, header validity, host-side validation.

No call here launches a kernel: every argument error is detected on the host
before the library touches the device.
"""
import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


@pytest.fixture(scope="module")
def lib():
    from tensor_sharded_mlp_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


@pytest.fixture(scope="module")
def b(lib):
    from tensor_sharded_mlp_b200 import binding
    return binding


def _declared():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(tp_mlp_\w+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("tp_mlp_create", "tp_mlp_forward", "tp_mlp_partials", "tp_mlp_destroy",
              "tp_mlp_pack", "tp_mlp_unpack", "tp_mlp_forward_packed", "tp_mlp_workspace_bytes",
              "tp_mlp_set_workspace", "tp_mlp_packed_bytes", "tp_mlp_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    nm = subprocess.run(["nm", "-D", "--defined-only", lib._name], capture_output=True, text=True,
                        check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\w+)$", nm, flags=re.M))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing


def test_binding_covers_every_symbol(b):
    assert set(_declared()) <= set(b.EXPORTED)


def test_header_compiles_as_c(tmp_path, lib):
    src = tmp_path / "use.c"
    src.write_text('#include "tp_mlp.h"\n#include <stdio.h>\n'
                   'int main(void){ tp_mlp_t h = 0;\n'
                   ' int s = tp_mlp_create(&h, 64, 256, 64, 2, TP_MLP_ACT_TANH, TP_MLP_F32, 4);\n'
                   ' printf("%d %zu %s\\n", s, tp_mlp_packed_bytes(h), tp_mlp_status_string(s));\n'
                   ' tp_mlp_destroy(h); return s; }\n')
    exe = tmp_path / "use"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), lib._name, "-Wl,-rpath," + os.path.dirname(lib._name)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    # part 1: 256 rows x 64 k = one block; part 2: 64 rows padded to a 256-row tile x 4 k-blocks
    assert out[0] == "0" and int(out[1]) == 256 * 64 * 4 + 256 * 256 * 4


def test_create_argument_errors(b):
    E = b.STATUS
    cases = [((64, 256, 64, 3, "tanh", "f32", 4), "ERR_SHAPE"),     # d_ff % tp
             ((64, 256, 64, 0, "tanh", "f32", 4), "ERR_SHAPE"),
             ((64, 256, 64, 16, "tanh", "f32", 4), "ERR_SHAPE"),    # tp > 8
             ((0, 256, 64, 2, "tanh", "f32", 4), "ERR_SHAPE"),
             ((64, 256, 64, 2, "tanh", "f32", 0), "ERR_SHAPE"),
             ((64, 256, 0, 2, "tanh", "f32", 4), "ERR_SHAPE")]
    for args, want in cases:
        with pytest.raises(b.TpMlpError) as ei:
            b.tp_mlp_create(*args)
        assert ei.value.name == want, args
    h = ctypes.c_void_p()
    assert b._lib.tp_mlp_create(ctypes.byref(h), 64, 256, 64, 2, 7, 0, 4) == 1   # bad act
    assert b._lib.tp_mlp_create(ctypes.byref(h), 64, 256, 64, 2, 0, 5, 4) == 1   # bad dtype
    assert b._lib.tp_mlp_create(None, 64, 256, 64, 2, 0, 0, 4) == 1


def test_sizes_follow_the_documented_layout(b):
    def a256(v):
        return (v + 255) // 256 * 256
    for act, dtype, d, f, dout, tp in [("tanh", "f32", 64, 256, 64, 2), ("swiglu", "bf16", 8192, 28672, 8192, 8),
                                       ("swiglu", "bf16", 40, 200, 24, 4), ("identity", "bf16", 8, 8, 4, 4)]:
        h = b.tp_mlp_create(d, f, dout, tp, act, dtype, 32)
        e = 4 if dtype == "f32" else 2
        rows1 = 256 * -(-f // 128) if act == "swiglu" else f

        def blocked(R, K):   # whole 256-row tiles x whole 64-wide k-blocks
            return -(-R // 256) * 256 * -(-K // 64) * 64
        assert b.tp_mlp_packed_bytes(h) == a256(blocked(rows1, d) * e) + a256(blocked(dout, f) * e)
        w = [b.tp_mlp_workspace_bytes(h, t) for t in range(0, 33)]
        assert all(x > 0 for x in w) and all(w[i] <= w[i + 1] for i in range(32))
        assert w[32] >= 32 * f * e            # holds H
        assert b.tp_mlp_workspace_bytes(h, 33) == 0
        b.tp_mlp_destroy(h)


def test_call_argument_errors_before_any_launch(b):
    """Each bad argument is rejected on the host (no device is present here)."""
    L = b._lib
    h = b.tp_mlp_create(64, 256, 64, 2, "tanh", "f32", 4)
    vp = ctypes.c_void_p
    arr = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    A = ctypes.cast(arr, b._vpp)
    ok_ptr = vp(0x100000)
    bad_ptr = vp(0x100004)         # not 16-byte aligned
    assert L.tp_mlp_forward(None, ok_ptr, 1, A, A, 2, 0, ok_ptr, None) == 1
    assert L.tp_mlp_forward(h, ok_ptr, 5, A, A, 2, 0, ok_ptr, None) == 2       # tokens > max
    assert L.tp_mlp_forward(h, ok_ptr, -1, A, A, 2, 0, ok_ptr, None) == 2
    assert L.tp_mlp_forward(h, ok_ptr, 1, A, A, 4, 0, ok_ptr, None) == 2       # tp mismatch
    assert L.tp_mlp_forward(h, ok_ptr, 1, A, A, 2, 1, ok_ptr, None) == 1       # act mismatch
    assert L.tp_mlp_forward(h, None, 1, A, A, 2, 0, ok_ptr, None) == 1          # null x
    assert L.tp_mlp_forward(h, bad_ptr, 1, A, A, 2, 0, ok_ptr, None) == 3       # misaligned
    assert L.tp_mlp_forward(h, ok_ptr, 0, A, A, 2, 0, ok_ptr, None) == 0        # 0 tokens: no-op
    assert L.tp_mlp_partials(h, ok_ptr, 1, A, A, 2, 0, None, None) == 1
    assert L.tp_mlp_forward_packed(h, ok_ptr, 5, ok_ptr, ok_ptr, None) == 2
    assert L.tp_mlp_forward_packed(h, bad_ptr, 1, ok_ptr, ok_ptr, None) == 3
    assert L.tp_mlp_pack(None, A, A, ok_ptr, None) == 1
    assert L.tp_mlp_set_plan(h, 10) == 1
    assert L.tp_mlp_set_plan(h, 9) == 0          # the fused skinny plan
    assert L.tp_mlp_set_plan(h, 3) == 0
    assert L.tp_mlp_forward_packed(h, ok_ptr, 1, ok_ptr, ok_ptr, None) == 4     # tcgen05 needs bf16
    assert L.tp_mlp_set_plan(h, 2) == 0
    assert L.tp_mlp_forward_packed(h, ok_ptr, 1, ok_ptr, ok_ptr, None) == 4     # GEMV needs bf16
    assert L.tp_mlp_set_plan(h, 0) == 0
    assert L.tp_mlp_set_workspace(h, ok_ptr, 16) == 7                           # too small
    assert L.tp_mlp_set_profile_events(h, None, 9) == 1
    assert L.tp_mlp_set_splitk(h, 4) == 1 and L.tp_mlp_set_splitk(h, -1) == 1
    assert L.tp_mlp_set_splitk(None, 0) == 1
    # fused all-reduce + residual + RMSNorm: argument checks come before any pointer use
    F = L.tp_mlp_allreduce_residual_rmsnorm
    assert F(None, 0, 1, 64, None, None, 0.0, 0, None, None, None) == 2       # tp_degree
    assert F(None, 2, 1, 62, None, None, 0.0, 0, None, None, None) == 2       # d % 4
    assert F(None, 2, 1, 49156, None, None, 0.0, 0, None, None, None) == 2    # too wide
    assert F(None, 2, 1, 64, None, None, -1.0, 0, None, None, None) == 1      # eps < 0
    assert F(None, 2, 1, 64, None, None, float("inf"), 0, None, None, None) == 1
    assert F(None, 2, 1, 64, None, None, 0.0, 7, None, None, None) == 1       # dtype
    assert F(None, 2, 1, 64, None, None, 0.0, 0, None, None, None) == 1       # null pointers
    assert F(None, 2, 0, 64, None, None, 0.0, 0, None, None, None) == 0       # no tokens: no-op
    # merge of attention partials
    M = L.tp_mlp_merge_attention_partials
    assert M(0, 4, 128, None, None, None, 0, None, None) == 2                  # tp_degree
    assert M(2, 4, 130, None, None, None, 0, None, None) == 2                  # head_dim % 4
    assert M(2, 4, 4100, None, None, None, 0, None, None) == 2                 # head_dim too large
    assert M(2, 4, 128, None, None, None, 3, None, None) == 1                  # dtype
    assert M(2, 4, 128, None, None, None, 1, None, None) == 1                  # null pointers
    assert M(2, 0, 128, None, None, None, 1, None, None) == 0                  # no rows: no-op
    # host<->device copy: these checks come before any driver query
    C = L.tp_mlp_copy_async
    assert C(ok_ptr, bad_ptr, 0, None) == 0                                    # no bytes: no-op
    assert C(ok_ptr, None, 64, None) == 1 and C(None, ok_ptr, 64, None) == 1   # null pointers
    assert C(ok_ptr, bad_ptr, 64, None) == 3 and C(bad_ptr, ok_ptr, 64, None) == 3
    for mode in (3, 2, 1, 0):
        assert L.tp_mlp_set_splitk(h, mode) == 0
    assert L.tp_mlp_last_plan(h) == 1 and L.tp_mlp_last_launches(h) == 0        # the 0-token no-op
    b.tp_mlp_destroy(h)
    for s in range(8):
        assert b.tp_mlp_status_string(s) not in ("", "unknown status")
    assert b.tp_mlp_status_string(99) == "unknown status"


def test_binding_pairs_shards_strictly(b):
    import torch
    h = b.tp_mlp_create(8, 8, 4, 2, "tanh", "f32", 2)
    t = torch.zeros(8, 4)
    with pytest.raises(ValueError):
        b.tp_mlp_forward(h, torch.zeros(1, 8), [t, t], [t], 2, "tanh", torch.zeros(1, 4))
    b.tp_mlp_destroy(h)


def test_binding_copy_checks_before_the_library(b):
    """The copy wrapper refuses mismatched sizes, strided tensors and pageable
    host tensors before calling the library (no device is present here)."""
    import torch
    with pytest.raises(ValueError):
        b.tp_mlp_copy_async(torch.zeros(16, dtype=torch.uint8), torch.zeros(32, dtype=torch.uint8))
    with pytest.raises(ValueError):
        b.tp_mlp_copy_async(torch.zeros(4, 4)[:, :2], torch.zeros(4, 2))
    with pytest.raises(ValueError):   # pageable (not pinned) host memory
        b.tp_mlp_copy_async(torch.zeros(64, dtype=torch.uint8), torch.zeros(64, dtype=torch.uint8))


def _model_slots(tiles, KB, BT, sms=148):
    """Split pieces per tile under the documented grid rule: floor(sms / tiles)
    CTAs per tile when that keeps 80 % of the SMs busy, else equal contiguous
    shares of the (tile, k-block) stream over every SM."""
    G = sms
    if tiles <= sms:
        s = min(sms // tiles, KB)
        if s >= 1 and 5 * tiles * s >= 4 * sms:
            G = tiles * s
    total = tiles * KB
    G = min(G, total)

    def owner(it):
        return ((it + 1) * G - 1) // total
    return max(owner(t * KB + KB - 1) - owner(t * KB) + 1 for t in range(tiles))


@pytest.mark.parametrize("act,d,f,dout,tp", [("tanh", 4096, 16384, 4096, 8), ("swiglu", 8192, 28672, 8192, 8),
                                             ("tanh", 512, 1024, 384, 4)])
def test_workspace_covers_every_skinny_tiling(b, act, d, f, dout, tp):
    """The split-tile scratch must hold the largest of every tiling the skinny
    path may pick (packed or shard form, 256- or 128-row tiles, either
    projection), since the split mode can change after the workspace is sized."""
    h = b.tp_mlp_create(d, f, dout, tp, act, "bf16", 128)
    fs = f // tp
    for T, BT in ((16, 16), (32, 32), (64, 64), (128, 128)):
        need = 0
        for proj in (0, 1):
            KB = -(-(d if proj == 0 else f) // 64)
            for raw in (False, True):
                for half in (False, True):
                    if half and proj == 0 and act == "swiglu":
                        continue
                    rows = 128 if half else 256
                    if proj == 1:
                        tiles = -(-dout // rows)
                    elif not raw:
                        tiles = -(-((2 * f) if act == "swiglu" else f) // rows)
                    else:
                        per = 128 if (act == "swiglu" or half) else 256
                        tiles = tp * -(-fs // per)
                    need = max(need, tiles * _model_slots(tiles, KB, BT) * rows * BT * 4)
        assert b.tp_mlp_workspace_bytes(h, T) >= T * f * 2 + need, (T, need)
    b.tp_mlp_destroy(h)
