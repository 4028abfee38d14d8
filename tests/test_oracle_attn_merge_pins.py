"""Pins for the oracle of the merge of partial attention results across KV shards.

Source: "LLM 推理并行化：先找瓶颈，再决定怎么切", §三 4) 上下文并行（CP）, decode
context parallelism: each rank reports a maximum, an exponential sum and a
weighted value sum per query; the merge rescales by exp(max - global max),
adds, and divides; the result equals attention over the unsplit history.

The pages' printed merged output [0.769627, 0.779901] cannot pin anything: the
inputs that produced it are not printed ("parity unpinned" by that value).
"""
import numpy as np
import pytest
import torch

import oracle


def _qkv(rows, n, D, seed, score_scale=1.0):
    r = np.random.default_rng(seed)
    q = (r.standard_normal((rows, D)) * score_scale).astype(np.float32)
    k = r.standard_normal((n, D)).astype(np.float32)
    v = r.standard_normal((n, D)).astype(np.float32)
    return q, k, v


def _split(q, k, v, cuts, scale):
    parts = [oracle.attention_partial(q, k[a:b], v[a:b], scale) for a, b in zip(cuts[:-1], cuts[1:])]
    m = np.stack([p[0] for p in parts])
    s = np.stack([p[1] for p in parts])
    w = np.stack([p[2] for p in parts])
    return m, s, w


def test_full_attention_is_torch_softmax_attention():
    """Library routine: torch softmax(q k^T * scale) v in float64."""
    q, k, v = _qkv(5, 37, 16, 1)
    sc = 16 ** -0.5
    ref = torch.softmax(torch.from_numpy(q).double() @ torch.from_numpy(k).double().T * sc, dim=-1) \
        @ torch.from_numpy(v).double()
    np.testing.assert_allclose(oracle.attention_full(q, k, v, sc), ref.numpy(), rtol=1e-12, atol=1e-13)


def test_partial_over_all_keys_normalises_to_full_attention():
    q, k, v = _qkv(4, 20, 8, 2)
    m, s, w = oracle.attention_partial(q, k, v, 0.5)
    np.testing.assert_allclose(w / s[:, None], oracle.attention_full(q, k, v, 0.5), rtol=1e-12, atol=1e-13)
    scores = (q.astype(np.float64) @ k.astype(np.float64).T) * 0.5
    np.testing.assert_array_equal(m, scores.max(axis=1))       # the local maximum is the row's maximum


@pytest.mark.parametrize("cuts", [(0, 64), (0, 10, 64), (0, 1, 2, 30, 64), (0, 8, 16, 24, 32, 40, 48, 56, 64),
                                  (0, 20, 20, 64)])            # the last has an empty rank
def test_merge_of_shards_is_attention_over_the_whole_history(cuts):
    """The pages' claim: cutting the KV history does not change the attention output."""
    q, k, v = _qkv(6, 64, 32, 3, score_scale=2.0)
    sc = 32 ** -0.5
    m, s, w = _split(q, k, v, cuts, sc)
    got = oracle.merge_attention_partials(m.astype(np.float32), s.astype(np.float32), w.astype(np.float32))
    ref = oracle.attention_full(q, k, v, sc)
    np.testing.assert_allclose(got, ref, rtol=2e-6, atol=2e-6)   # fp32 rounding of the partials only


def test_one_rank_is_weighted_sum_over_exp_sum_exactly():
    r = np.random.default_rng(4)
    m = r.standard_normal((1, 7)).astype(np.float32)
    s = (1 + r.random((1, 7)) * 9).astype(np.float32)
    w = r.standard_normal((1, 7, 12)).astype(np.float32)
    got = oracle.merge_attention_partials(m, s, w)
    np.testing.assert_array_equal(got, w[0].astype(np.float64) / s[0].astype(np.float64)[:, None])


def test_equal_maxima_closed_form():
    """Equal maxima: every scale is 1, so the merge is (sum of w) / (sum of s)."""
    m = np.zeros((3, 2), np.float32)
    s = np.array([[1, 2], [3, 4], [5, 6]], np.float32)
    w = np.arange(3 * 2 * 4, dtype=np.float32).reshape(3, 2, 4)
    got = oracle.merge_attention_partials(m, s, w)
    np.testing.assert_allclose(got, w.astype(np.float64).sum(0) / s.astype(np.float64).sum(0)[:, None], rtol=1e-15)


def test_common_shift_of_the_maxima_changes_nothing_and_huge_scores_do_not_overflow():
    """Only differences of maxima matter; maxima near 1000 (where exp overflows
    without the global-maximum subtraction) merge to the same finite result."""
    r = np.random.default_rng(5)
    m = (np.round(r.standard_normal((4, 9)) * 8) / 8).astype(np.float32)   # on a 1/8 grid: shifts stay exact
    s = (1 + r.random((4, 9)) * 5).astype(np.float32)
    w = r.standard_normal((4, 9, 8)).astype(np.float32)
    base = oracle.merge_attention_partials(m, s, w)
    for shift in (1000.0, -1000.0, 64.0):
        shifted = (m + np.float32(shift)).astype(np.float32)
        assert np.array_equal(shifted.astype(np.float64) - shift, m.astype(np.float64))
        got = oracle.merge_attention_partials(shifted, s, w)
        np.testing.assert_array_equal(got, base)


def test_rank_order_does_not_matter():
    q, k, v = _qkv(3, 40, 8, 6)
    m, s, w = _split(q, k, v, (0, 7, 19, 40), 0.3)
    m, s, w = m.astype(np.float32), s.astype(np.float32), w.astype(np.float32)
    a = oracle.merge_attention_partials(m, s, w)
    perm = [2, 0, 1]
    b = oracle.merge_attention_partials(m[perm], s[perm], w[perm])
    np.testing.assert_allclose(a, b, rtol=1e-14, atol=1e-15)


def test_empty_ranks_contribute_nothing_and_all_empty_rows_are_zero():
    r = np.random.default_rng(7)
    m = r.standard_normal((2, 3)).astype(np.float32)
    s = (1 + r.random((2, 3))).astype(np.float32)
    w = r.standard_normal((2, 3, 4)).astype(np.float32)
    base = oracle.merge_attention_partials(m, s, w)
    m2 = np.concatenate([m, np.full((1, 3), -np.inf, np.float32)])
    s2 = np.concatenate([s, np.zeros((1, 3), np.float32)])
    w2 = np.concatenate([w, np.zeros((1, 3, 4), np.float32)])
    np.testing.assert_array_equal(oracle.merge_attention_partials(m2, s2, w2), base)
    empty = oracle.merge_attention_partials(np.full((2, 3), -np.inf, np.float32), np.zeros((2, 3), np.float32),
                                            np.zeros((2, 3, 4), np.float32))
    assert np.all(empty == 0.0)


def test_argument_errors():
    with pytest.raises(ValueError):
        oracle.merge_attention_partials(np.zeros((2, 3), np.float32), np.zeros((2, 4), np.float32),
                                        np.zeros((2, 3, 4), np.float32))
    with pytest.raises(ValueError):
        oracle.attention_full(np.zeros((1, 4), np.float32), np.zeros((0, 4), np.float32),
                              np.zeros((0, 4), np.float32), 1.0)
