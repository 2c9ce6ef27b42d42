"""Pins for the indexer-score oracle (CPU only).

Checked against a hand-worked example (tests/golden), closed forms (zero
queries; one-hot keys and queries) and invariants (head permutation, exact
power-of-two scaling of w, additivity over a split of the heads, permutation of
the keys, valid_len truncation).  Mutated copies of the scoring rule (ReLU
after the weight, ReLU after the head sum, no ReLU, transposed operands) are
shown to fail the worked example.
"""

import json
import os

import numpy as np
import pytest

from oracle import indexer_scores, indexer_topk, decode_bf16
from sparse_attention_top_ds_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(a):
    return inputs.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def load_example():
    with open(os.path.join(GOLDEN, "indexer_worked_example.json")) as f:
        return json.load(f)


def test_worked_example_scores_and_selection():
    ex = load_example()
    q, keys = bf16(ex["q"]), bf16(ex["keys"])
    for case in ex["cases"]:
        w = np.array(case["w"], dtype=np.float32)
        vl = None if case["valid_len"] is None else np.array(case["valid_len"])
        s = indexer_scores(q, keys, w, vl)[0]
        for got, want in zip(s, case["scores"]):
            if want is None:
                assert np.isnan(got)
            else:
                assert got == want
        for k, want in case["topk"].items():
            idx, _ = indexer_topk(q, keys, w, int(k), vl)
            m = sum(1 for e in want if e >= 0)
            assert sorted(idx[0, :m].tolist()) == sorted(e for e in want if e >= 0)
            assert idx[0, m:].tolist() == [-1] * (int(k) - m)


def test_zero_queries_give_zero_scores_and_lowest_indices():
    _, keys, w = inputs.indexer_factors(seed=2, batch=2, n=300, heads=8, d=128)
    q = np.zeros((2, 8, 128), dtype=np.uint16)
    s = indexer_scores(q, keys, w)
    assert np.all(s == 0.0)
    idx, _ = indexer_topk(q, keys, w, 17)
    assert idx.tolist() == [list(range(17))] * 2


def test_one_hot_closed_form():
    # k[s] = a_s e_j and q[t,h] = b_h e_j give q.k = a_s b_h, so
    # score[s] = relu(a_s) * P + relu(-a_s) * N with
    # P = sum_{b_h > 0} w_h b_h and N = sum_{b_h < 0} w_h (-b_h).
    H, d, S, j = 6, 128, 40, 77
    a = np.arange(S, dtype=np.float32) - 17.0                  # exact in bf16
    b = np.array([1.0, -2.0, 0.5, 3.0, -0.25, 0.0], dtype=np.float32)
    w = np.array([[0.75, 0.5, 2.0, 0.125, 4.0, 9.0]], dtype=np.float32)
    keys = np.zeros((S, d), dtype=np.float32)
    keys[:, j] = a
    q = np.zeros((1, H, d), dtype=np.float32)
    q[0, :, j] = b
    P = 0.75 * 1.0 + 2.0 * 0.5 + 0.125 * 3.0
    N = 0.5 * 2.0 + 4.0 * 0.25
    s = indexer_scores(bf16(q), bf16(keys), w)[0]
    expect = np.where(a > 0, a * P, -a * N).astype(np.float64)
    assert np.array_equal(s, expect)
    idx, _ = indexer_topk(bf16(q), bf16(keys), w, 5)
    # largest: a = 22, 21, 20, 19 -> 22*P.. vs a = -17 -> 17*N = 34 ; P = 2.125
    ranked = sorted(range(S), key=lambda i: (-expect[i], i))
    assert idx[0].tolist() == ranked[:5]


def _random_case(seed, batch=3, heads=8, S=257):
    q, keys, w = inputs.indexer_factors(seed=seed, batch=batch, n=S, heads=heads, d=128)
    return q, keys, w


def test_head_permutation_invariance():
    q, keys, w = _random_case(21)
    perm = np.random.default_rng(0).permutation(q.shape[1])
    a = indexer_scores(q, keys, w)
    b = indexer_scores(q[:, perm], keys, w[:, perm])
    assert np.allclose(a, b, rtol=1e-13, atol=0)


def test_power_of_two_weight_scaling_is_exact():
    q, keys, w = _random_case(22)
    a = indexer_scores(q, keys, w)
    b = indexer_scores(q, keys, (w.astype(np.float64) * 4.0))
    assert np.array_equal(b, 4.0 * a)


def test_additivity_over_head_split():
    q, keys, w = _random_case(23, heads=10)
    full = indexer_scores(q, keys, w)
    lo = indexer_scores(q[:, :3], keys, w[:, :3])
    hi = indexer_scores(q[:, 3:], keys, w[:, 3:])
    assert np.allclose(full, lo + hi, rtol=1e-12, atol=1e-15)


def test_key_permutation_permutes_scores():
    q, keys, w = _random_case(24)
    perm = np.random.default_rng(1).permutation(keys.shape[0])
    a = indexer_scores(q, keys, w)
    b = indexer_scores(q, keys[perm], w)
    assert np.allclose(a[:, perm], b, rtol=1e-13, atol=0)


def test_valid_len_is_a_prefix():
    q, keys, w = _random_case(25)
    vl = np.array([0, 100, 257])
    a = indexer_scores(q, keys, w)
    b = indexer_scores(q, keys, w, vl)
    assert np.all(np.isnan(b[0]))
    assert np.allclose(b[1, :100], a[1, :100], rtol=1e-13, atol=0) and np.all(np.isnan(b[1, 100:]))
    assert np.allclose(b[2], a[2], rtol=1e-13, atol=0)
    idx, _ = indexer_topk(q, keys, w, 150, vl)
    assert np.all(idx[0] == -1)
    assert np.all(idx[1, 100:] == -1) and np.all((idx[1, :100] >= 0) & (idx[1, :100] < 100))


def test_nonnegative_weights_give_nonnegative_scores():
    q, keys, w = _random_case(26)
    assert np.all(indexer_scores(q, keys, w) >= 0.0)


# ---------------------------------------------------------------- planted mistakes

def _m_relu_after_weight(q, k, w):
    d = decode_bf16(q)[0] @ decode_bf16(k).T
    return np.maximum(w[0][:, None] * d, 0).sum(0)


def _m_relu_after_sum(q, k, w):
    d = decode_bf16(q)[0] @ decode_bf16(k).T
    return np.maximum((w[0][:, None] * d).sum(0), 0)


def _m_no_relu(q, k, w):
    d = decode_bf16(q)[0] @ decode_bf16(k).T
    return (w[0][:, None] * d).sum(0)


def _m_transposed_keys(q, k, w):
    kk = decode_bf16(k)
    d = decode_bf16(q)[0][:, :kk.shape[0]] @ kk[:, :kk.shape[0]]   # keys used column-wise
    return (w[0][:, None] * np.maximum(d, 0)).sum(0)


@pytest.mark.parametrize("mutant", [_m_relu_after_weight, _m_relu_after_sum, _m_no_relu,
                                    _m_transposed_keys])
def test_worked_example_catches_planted_mistakes(mutant):
    ex = load_example()
    q, keys = bf16(ex["q"]), bf16(ex["keys"])
    wrong = False
    for case in ex["cases"]:
        if case["valid_len"] is not None:
            continue
        w = np.array(case["w"], dtype=np.float64)
        try:
            got = mutant(q, keys, w)
        except ValueError:
            wrong = True
            continue
        if got.shape != (5,) or not np.array_equal(got, np.array(case["scores"])):
            wrong = True
    assert wrong


def test_per_row_caches_equal_one_cache_per_call():
    q, keys, w = _random_case(27, batch=3, S=200)
    g = np.random.default_rng(3)
    kc3 = np.stack([keys, keys[g.permutation(200)], keys[::-1].copy()])
    vl = np.array([200, 57, 130])
    got = indexer_scores(q, kc3, w, vl)
    for t in range(3):
        one = indexer_scores(q[t:t + 1], kc3[t], w[t:t + 1], vl[t:t + 1])
        assert np.array_equal(np.nan_to_num(got[t], nan=-1.0), np.nan_to_num(one[0], nan=-1.0))
    idx, _ = indexer_topk(q, kc3, w, 20, vl)
    for t in range(3):
        i1, _ = indexer_topk(q[t:t + 1], kc3[t], w[t:t + 1], 20, vl[t:t + 1])
        assert idx[t].tolist() == i1[0].tolist()
