"""Host-side checks: the seeded input generator and the analytic counts."""
import json
import os

import numpy as np
import pytest
import torch

from tensor_sharded_mlp_b200 import counts, inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_counts.json")


def test_generator_is_deterministic_and_ordered():
    p1 = inputs.generate(3, 16, 32, "swiglu", "bf16", seed=5, init=0.02)
    p2 = inputs.generate(3, 16, 32, "swiglu", "bf16", seed=5, init=0.02)
    for k in ("x", "gate", "up", "b"):
        assert np.array_equal(getattr(p1, k), getattr(p2, k))
    # draw order X, gate, up, down from one stream
    r = np.random.default_rng(5)
    x = r.standard_normal((3, 16))
    g = r.standard_normal((16, 32)) * 0.02
    assert np.array_equal(p1.x, inputs.round_to_bf16(x.astype(np.float32)))
    assert np.array_equal(p1.gate, inputs.round_to_bf16(g.astype(np.float32)))


def test_chunked_draw_matches_single_draw(monkeypatch):
    monkeypatch.setattr(inputs, "_CHUNK_ELEMS", 100)
    p = inputs.generate(2, 40, 64, "tanh", "f32", seed=9)
    r = np.random.default_rng(9)
    r.standard_normal((2, 40))
    a = (r.standard_normal((40, 64)) * 40 ** -0.5).astype(np.float32)
    assert np.array_equal(p.a, a)


def test_bf16_rounding_matches_torch():
    r = np.random.default_rng(0)
    v = (r.standard_normal(100000) * np.exp(r.uniform(-20, 20, 100000))).astype(np.float32)
    v = np.concatenate([v, np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0],
                                    np.float32)])
    ours = inputs.round_to_bf16(v)
    theirs = torch.from_numpy(v).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours, theirs)
    # ties to even: 1 + 2^-8 is halfway between 1 and 1 + 2^-7 -> 1
    assert ours[-4] == 1.0 and ours[-3] == np.float32(1.0 + 2 ** -6)


def test_shards_concatenate_back_bit_exact():
    """Column shards concatenate to A; row shards stack to B ([vLLM] §1.2.3)."""
    for act in ("tanh", "swiglu"):
        p = inputs.generate(2, 8, 32, act, "bf16", seed=1)
        for tp in (1, 2, 4, 8):
            A, B = p.shards(tp)
            fs = 32 // tp
            assert len(A) == len(B) == tp
            assert np.array_equal(np.vstack(B), p.b)
            if act == "swiglu":
                assert np.array_equal(np.hstack([a[:, :fs] for a in A]), p.gate)
                assert np.array_equal(np.hstack([a[:, fs:] for a in A]), p.up)
            else:
                assert np.array_equal(np.hstack(A), p.a)
    with pytest.raises(ValueError):
        inputs.generate(1, 8, 30, "tanh").shards(4)


def test_sample_rows_sorted_distinct():
    p = inputs.generate(50, 4, 8, "tanh", seed=2)
    rows = p.sample_rows(10)
    assert len(set(rows.tolist())) == 10 and np.all(np.diff(rows) > 0)


def test_counts_match_page_figures():
    g = json.load(open(GOLDEN))
    d = g["decode_70b_fp16"]
    # 2N FLOPs per token and N * bytes weights ([7.4] §7.4.1)
    assert 2 * d["params"] == d["flops_per_token"]
    assert d["params"] * d["bytes_per_param"] == d["weight_bytes"]
    c = g["tp_columns_per_rank"]
    for tp, n in c["per_rank"].items():
        assert counts.columns_per_rank(c["columns"], int(tp)) == n
        p = inputs.generate(1, 4, c["columns"], "tanh", seed=0)
        A, B = p.shards(int(tp))
        assert all(a.shape[1] == n for a in A) and all(b.shape[0] == n for b in B)
    m = g["allreduce_message_decode"]
    assert counts.allreduce_bytes(m["batch"], m["seq"], m["d_model"], m["bytes_per_elem"]) == m["bytes"]


def test_counts_for_decode_config():
    c = inputs.CONFIGS["decode_bs1"]
    N = counts.mlp_params(c["d_model"], c["d_ff"], c["d_model"], "swiglu")
    assert N == 3 * 8192 * 28672
    assert counts.weight_bytes(8192, 28672, 8192, "swiglu", "bf16") == 1409286144
    assert counts.forward_flops(1, 8192, 28672, 8192, "swiglu") == 2 * N
    assert (counts.gemm1_flops(7, 8192, 28672, "swiglu") + counts.gemm2_flops(7, 28672, 8192)
            == counts.forward_flops(7, 8192, 28672, 8192, "swiglu"))
    tot = counts.algorithmic_bytes(32, 8192, 28672, 8192, "swiglu", "bf16")
    assert tot == counts.gemm1_bytes(32, 8192, 28672, "swiglu", "bf16") + \
        counts.gemm2_bytes(32, 28672, 8192, "bf16")


def test_fused_norm_inputs_are_seeded_and_dtype_exact():
    a = inputs.generate_fused_norm(3, 16, 2, "bf16", seed=4)
    b = inputs.generate_fused_norm(3, 16, 2, "bf16", seed=4)
    assert a.partials.shape == (2, 3, 16) and a.residual.shape == (3, 16) and a.gamma.shape == (16,)
    for x, y in ((a.partials, b.partials), (a.residual, b.residual), (a.gamma, b.gamma)):
        assert x.dtype == np.float32 and np.array_equal(x, y)
    # residual and gamma hold bf16 values; the fp32 partials are not rounded
    assert np.array_equal(a.residual, inputs.round_to_bf16(a.residual))
    assert np.array_equal(a.gamma, inputs.round_to_bf16(a.gamma))
    assert not np.array_equal(a.partials, inputs.round_to_bf16(a.partials))
    assert not np.array_equal(a.partials, inputs.generate_fused_norm(3, 16, 2, "bf16", seed=5).partials)


def test_attn_merge_inputs_are_seeded_and_in_range():
    a = inputs.generate_attn_merge(4, 10, 8, "bf16", seed=7, keys_per_rank=64)
    assert a.maximum.shape == (4, 10) and a.exp_sum.shape == (4, 10) and a.weighted.shape == (4, 10, 8)
    assert np.all(a.exp_sum >= 1.0) and np.all(a.exp_sum <= 64.0)   # at least the maximum's own term
    assert np.array_equal(a.weighted, inputs.round_to_bf16(a.weighted))
    b = inputs.generate_attn_merge(4, 10, 8, "bf16", seed=7, keys_per_rank=64)
    assert np.array_equal(a.weighted, b.weighted) and np.array_equal(a.maximum, b.maximum)


def test_fused_norm_byte_counts():
    # 2 ranks, 3 tokens, width 4, bf16: partials 2*3*4*4, residual 3*4*2, gamma 4*2, outputs 2*3*4*2
    assert counts.fused_norm_bytes(2, 3, 4, "bf16") == 96 + 24 + 8 + 48
    # unfused: Z and h each written and read once more (2 * 2 * n * e)
    assert counts.unfused_norm_bytes(2, 3, 4, "bf16") - counts.fused_norm_bytes(2, 3, 4, "bf16") == 2 * 2 * 12 * 2


def test_kernel_source_hash_ignores_comments_only():
    code = "int f(int a) { return a + 1; }"
    assert counts._code_only("// lead\nint f(int a) {  /* note */ return a + 1; }  // tail") == code
    assert counts._code_only(code) != counts._code_only(code.replace("+ 1", "+ 2"))
