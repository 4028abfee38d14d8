"""GPU parity of the merge of partial attention results across KV shards.

"LLM 推理并行化：先找瓶颈，再决定怎么切", §三 4) 上下文并行（CP）, decode context
parallelism.  Partials come from the oracle's rank-local step over random
q, K, V (so the merge must also reproduce attention over the whole history)
and from the seeded generator; edge cases cover empty ranks, rows with every
rank empty, maxima near +-1000, head sizes that share a warp between rows
(with a ragged last warp), that leave some of a row's lanes idle or give
them one group more than the others, that rule out 16-byte bf16 loads
(head_dim % 8 != 0), the largest head size the kernel takes, and row counts
of several waves of CTAs with a ragged last one.
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


def _merge(m, s, w, dtype):
    out = B().tp_mlp_merge_attention_partials(torch.from_numpy(np.ascontiguousarray(m)).cuda(),
                                              torch.from_numpy(np.ascontiguousarray(s)).cuda(), dev(w, dtype))
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("cuts", [(0, 96), (0, 40, 96), (0, 12, 12, 50, 96), (0, 12, 24, 36, 48, 60, 72, 84, 96)])
def test_merge_reproduces_attention_over_the_whole_history(cuts):
    r = np.random.default_rng(len(cuts))
    rows, n, D = 24, 96, 64
    q = (r.standard_normal((rows, D)) * 2).astype(np.float32)
    k = r.standard_normal((n, D)).astype(np.float32)
    v = r.standard_normal((n, D)).astype(np.float32)
    sc = D ** -0.5
    parts = [oracle.attention_partial(q, k[a:b], v[a:b], sc) for a, b in zip(cuts[:-1], cuts[1:])]
    m = np.stack([p[0] for p in parts]).astype(np.float32)
    s = np.stack([p[1] for p in parts]).astype(np.float32)
    w = np.stack([p[2] for p in parts]).astype(np.float32)
    got = _merge(m, s, w, "f32")
    assert_close(got, oracle.merge_attention_partials(m, s, w), "f32", "merge vs merge oracle")
    assert_close(got, oracle.attention_full(q, k, v, sc), "f32", "merge vs full attention")


SHAPES = [(1, 1, 4), (2, 3, 64), (3, 5, 68), (8, 2048, 128), (5, 33, 132), (8, 100, 4096), (7, 9, 256),
          (4, 37, 8), (6, 50, 24), (2, 300, 40), (8, 65, 12)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("P,rows,D", SHAPES)
def test_merge_parity(P, rows, D, dtype):
    a = inputs.generate_attn_merge(P, rows, D, dtype, seed=P * 100 + rows + D)
    got = _merge(a.maximum, a.exp_sum, a.weighted, dtype)
    assert_close(got, oracle.merge_attention_partials(a.maximum, a.exp_sum, a.weighted), dtype,
                 f"merge P={P} rows={rows} D={D}")


# many rows: several waves of CTAs, ragged last CTAs
MANY_ROWS = [(8, 16384 + 5, 128), (2, 40000, 64), (4, 77777, 136), (8, 9999, 256), (1, 300001, 16)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("P,rows,D", MANY_ROWS)
def test_merge_parity_many_rows(P, rows, D, dtype):
    a = inputs.generate_attn_merge(P, rows, D, dtype, seed=P + rows + D)
    got = _merge(a.maximum, a.exp_sum, a.weighted, dtype)
    assert_close(got, oracle.merge_attention_partials(a.maximum, a.exp_sum, a.weighted), dtype,
                 f"merge P={P} rows={rows} D={D}")


def test_empty_ranks_and_rows_and_huge_maxima():
    a = inputs.generate_attn_merge(4, 40, 128, "f32", seed=9)
    m, s, w = a.maximum.copy(), a.exp_sum.copy(), a.weighted.copy()
    m[1, :10] = -np.inf                  # rank 1 has no keys for rows 0..9
    s[1, :10] = 0.0
    w[1, :10] = 0.0
    m[:, 20] = -np.inf                   # row 20: every rank empty
    s[:, 20] = 0.0
    w[:, 20] = 0.0
    m[:, 30:] += np.float32(1000.0)      # rows 30..: scores where exp would overflow unshifted
    got = _merge(m, s, w, "f32")
    ref = oracle.merge_attention_partials(m, s, w)
    assert torch.isfinite(got).all()
    assert torch.all(got[20] == 0)
    assert_close(got, ref, "f32", "edge cases")


def test_no_rows_is_a_no_op():
    z = torch.zeros(3, 0, device="cuda")
    out = B().tp_mlp_merge_attention_partials(z, z, torch.zeros(3, 0, 64, device="cuda"))
    assert out.shape == (0, 64)


def test_merge_rejects_bad_arguments_before_launch():
    a = inputs.generate_attn_merge(2, 4, 64, "f32", seed=3)
    m = torch.from_numpy(a.maximum).cuda()
    s = torch.from_numpy(a.exp_sum).cuda()
    w = torch.from_numpy(a.weighted).cuda()
    out = torch.empty(4, 64, device="cuda")
    L, ptr = B()._lib, B()._ptr
    assert L.tp_mlp_merge_attention_partials(2, 4, 64, ptr(m), ptr(s), ptr(w), 0, ptr(out), None) == 0
    torch.cuda.synchronize()
    # buffers claimed larger than their allocation (past the allocator's 2 MB segment)
    assert L.tp_mlp_merge_attention_partials(2, 100000, 64, ptr(m), ptr(s), ptr(w), 0, ptr(out), None) == 2
    misaligned = B().ctypes.c_void_p(w.data_ptr() + 8)
    assert L.tp_mlp_merge_attention_partials(2, 4, 64, ptr(m), ptr(s), misaligned, 0, ptr(out), None) == 3


@pytest.mark.parametrize("name", ["attn_merge_decode_bs32", "attn_merge_decode_bs256"])
def test_merge_bench_configs_full_size(name):
    """The workloads bench.py times, at their full sizes, every row checked."""
    c = inputs.ATTN_MERGE_CONFIGS[name]
    a = inputs.generate_attn_merge(c["tp"], c["tokens"] * c["heads"], c["head_dim"], c["dtype"], c["seed"],
                                   c["keys_per_rank"])
    got = _merge(a.maximum, a.exp_sum, a.weighted, c["dtype"])
    assert_close(got, oracle.merge_attention_partials(a.maximum, a.exp_sum, a.weighted), c["dtype"], name)
