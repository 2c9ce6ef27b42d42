"""Pins for the indexer query projection oracle (CPU only).

Checked against closed forms (one-hot inputs pick out one weight column;
a hand-worked 2-token example), invariants (linearity in x, exact power-of-two
scaling, head permutation) and, for the bfloat16 rounding, against the input
generator's independent float32 -> bfloat16 rounding.  A planted mistake
(transposed weights, a dropped head offset) is shown to fail the pins.
"""

import numpy as np
import pytest

from oracle import qproj, round_bf16
from sparse_attention_top_ds_b200 import inputs


def bf16(a):
    return inputs.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _dec(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_worked_example():
    # 2 tokens, d_in = 3, 1 head of d = 2 (so Wq has 2 rows) and Ww one row:
    # q[0] = [1*1 + 2*0 + 3*(-1), 1*0.5 + 2*0.25 + 3*0] = [-2, 1]
    # q[1] = [0*1 + (-1)*0 + 4*(-1), 0*0.5 + (-1)*0.25 + 4*0] = [-4, -0.25]
    # w[0] = 1*2 + 2*0 + 3*1 = 5 ; w[1] = 0*2 + (-1)*0 + 4*1 = 4
    x = bf16([[1, 2, 3], [0, -1, 4]])
    wq = bf16([[1, 0, -1], [0.5, 0.25, 0]])
    ww = bf16([[2, 0, 1]])
    q, w = qproj(x, wq, ww, heads=1, d=2)
    assert q.tolist() == [[[-2.0, 1.0]], [[-4.0, -0.25]]]
    assert w.tolist() == [[5.0], [4.0]]


def test_one_hot_input_picks_a_column():
    g = np.random.default_rng(1)
    d_in, H = 40, 3
    wq = bf16(g.standard_normal((H * 128, d_in)))
    ww = bf16(g.standard_normal((H, d_in)))
    for i in (0, 17, 39):
        x = np.zeros((1, d_in), dtype=np.float32)
        x[0, i] = 1.0
        q, w = qproj(bf16(x), wq, ww)
        assert np.array_equal(q.reshape(-1), _dec(wq)[:, i])
        assert np.array_equal(w.reshape(-1), _dec(ww)[:, i])


def test_linearity_and_exact_scaling():
    g = np.random.default_rng(2)
    T, d_in, H = 3, 64, 2
    wq = bf16(g.standard_normal((H * 128, d_in)))
    x1 = bf16(g.standard_normal((T, d_in)))
    x2 = bf16(g.standard_normal((T, d_in)))
    s = bf16(_dec(x1) + _dec(x2))              # rounded sum, compared through its own decode
    q1, _ = qproj(x1, wq)
    q2, _ = qproj(x2, wq)
    qs, _ = qproj(s, wq)
    lin = qproj(bf16(_dec(x1) * 4.0), wq)[0]
    assert np.array_equal(lin, 4.0 * q1)        # exact: a power of two
    exact_sum = np.einsum("ti,ni->tn", _dec(x1) + _dec(x2), _dec(wq)).reshape(qs.shape)
    assert np.allclose(q1 + q2, exact_sum, rtol=1e-12, atol=1e-12)
    assert np.allclose(qs, np.einsum("ti,ni->tn", _dec(s), _dec(wq)).reshape(qs.shape), rtol=1e-12, atol=1e-12)


def test_head_permutation():
    g = np.random.default_rng(3)
    T, d_in, H = 2, 32, 4
    wq = bf16(g.standard_normal((H * 128, d_in)))
    ww = bf16(g.standard_normal((H, d_in)))
    x = bf16(g.standard_normal((T, d_in)))
    perm = np.array([2, 0, 3, 1])
    q, w = qproj(x, wq, ww)
    qp, wp = qproj(x, wq.reshape(H, 128, d_in)[perm].reshape(H * 128, d_in), ww[perm])
    assert np.array_equal(qp, q[:, perm]) and np.array_equal(wp, w[:, perm])


def test_round_bf16_matches_the_generators_rounding():
    g = np.random.default_rng(4)
    v = np.concatenate([g.standard_normal(20000) * 10.0 ** g.integers(-8, 8, 20000),
                        [1.0, -1.0, 2.0 ** -100, 3.0 * 2 ** 60]]).astype(np.float32)
    # ties: values halfway between two bfloat16 numbers, both parities
    base = _dec(bf16(g.standard_normal(2000)))
    ulp = 2.0 ** (np.floor(np.log2(np.abs(base))) - 7)
    ties = (base + ulp / 2).astype(np.float32)
    for arr in (v, ties):
        ref = _dec(bf16(arr))
        got = round_bf16(arr.astype(np.float64))
        assert np.array_equal(got, ref)


def test_round_bf16_subnormals_and_overflow():
    g = np.random.default_rng(5)
    # bfloat16 subnormals (below 2^-126, quantum 2^-133), values halfway between
    # two of them, and the boundary to the normal range
    sub = (g.standard_normal(5000) * 2.0 ** -131).astype(np.float32)
    kk = g.integers(-127, 128, 500).astype(np.float64)
    sub_ties = ((kk + 0.5) * 2.0 ** -133).astype(np.float32)
    edge = np.array([2.0 ** -126, 2.0 ** -126 - 2.0 ** -134, 2.0 ** -134, -2.0 ** -134, 3 * 2.0 ** -134,
                     2.0 ** -149], dtype=np.float32)
    # the top: the largest finite bfloat16, the tie above it (rounds to even:
    # infinity), and the largest float32
    big = (2.0 - 2.0 ** -7) * 2.0 ** 127
    top = np.array([big, -big, big + 2.0 ** 118, (2.0 - 2.0 ** -8) * 2.0 ** 127, 3.4028234663852886e38],
                   dtype=np.float32)
    for arr in (sub, sub_ties, edge, top):
        ref = _dec(bf16(arr))
        got = round_bf16(arr.astype(np.float64))
        assert np.array_equal(got, ref)
        assert np.array_equal(np.signbit(got), np.signbit(ref))
    assert np.isinf(round_bf16(np.array([(2.0 - 2.0 ** -8) * 2.0 ** 127]))[0])
    assert round_bf16(np.array([big]))[0] == big


def _correct(x, wq, heads, d):
    return qproj(x, wq, heads=heads, d=d)[0]


def _m_head0_everywhere(x, wq, heads, d):
    # every head uses the first head's rows (a dropped head offset)
    xx, ww = _dec(x), _dec(wq)
    return np.stack([np.stack([ww[:d] @ xx[t] for _ in range(heads)]) for t in range(xx.shape[0])])


def _m_row_major_confusion(x, wq, heads, d):
    # output feature n read as column n of Wq viewed as [d_in, heads*d]
    xx, ww = _dec(x), _dec(wq)
    w2 = ww.reshape(-1)[: xx.shape[1] * heads * d].reshape(xx.shape[1], heads * d)
    return (xx @ w2).reshape(xx.shape[0], heads, d)


def _pins_pass(fn):
    x = bf16([[1, 2, 3], [0, -1, 4]])
    wq = bf16([[1, 0, -1], [0.5, 0.25, 0]])
    if fn(x, wq, 1, 2).tolist() != [[[-2.0, 1.0]], [[-4.0, -0.25]]]:
        return False
    g = np.random.default_rng(1)
    d_in, H = 40, 3
    wq = bf16(g.standard_normal((H * 128, d_in)))
    for i in (0, 17, 39):
        x = np.zeros((1, d_in), dtype=np.float32)
        x[0, i] = 1.0
        if not np.array_equal(fn(bf16(x), wq, H, 128).reshape(-1), _dec(wq)[:, i]):
            return False
    return True


def test_pins_accept_the_oracle():
    assert _pins_pass(_correct)


@pytest.mark.parametrize("mutant", [_m_head0_everywhere, _m_row_major_confusion])
def test_pins_catch_planted_mistakes(mutant):
    assert not _pins_pass(mutant)
