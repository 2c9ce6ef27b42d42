"""Pins for the compressor-fold oracle (CPU only).

PARITY UNPINNED with respect to the pages, which do not give the gate: these
pins check the oracle against the closed forms of its stated reading
(s_i = g . x_i, a = softmax(s), out = sum a_i x_i), so that a slip in the
arithmetic (a dropped normalisation, a transposed product, the wrong axis of
the softmax) still shows.
"""

import math

import numpy as np
import pytest

from oracle import compress_fold
from sparse_attention_top_ds_b200 import inputs


def bf16(a):
    return inputs.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _dec(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_worked_example():
    # D = 2, gate (1, 0): scores are the first channels 0, 1, 2, 3; weights e^i / S
    # with S = 1 + e + e^2 + e^3; out[1] = sum_i w_i * 1 = 1.
    x = bf16([[[0, 1], [1, 1], [2, 1], [3, 1]]])
    out = compress_fold(x, bf16([1, 0]))
    S = 1 + math.e + math.e ** 2 + math.e ** 3
    assert out[0, 0] == pytest.approx((math.e + 2 * math.e ** 2 + 3 * math.e ** 3) / S, abs=1e-14)
    assert out[0, 1] == pytest.approx(1.0, abs=1e-15)


def test_zero_gate_is_the_mean():
    g = np.random.default_rng(1)
    x = bf16(g.standard_normal((3, 4, 64)))
    out = compress_fold(x, np.zeros(64, dtype=np.uint16))
    assert np.allclose(out, _dec(x).mean(axis=1), rtol=1e-14, atol=1e-15)


def test_equal_rows_fold_to_the_row():
    g = np.random.default_rng(2)
    row = bf16(g.standard_normal(32))
    x = np.tile(row, (2, 4, 1))
    out = compress_fold(x, bf16(g.standard_normal(32)))
    assert np.allclose(out, np.tile(_dec(row), (2, 1)), rtol=1e-14, atol=1e-15)


def test_a_dominant_score_picks_its_token():
    g = np.random.default_rng(3)
    x = _dec(bf16(g.standard_normal((1, 4, 16))))
    x[0, 2, 0] = 64.0                      # gate on channel 0 makes token 2's score 64, the others < 5
    gate = np.zeros(16)
    gate[0] = 1.0
    out = compress_fold(bf16(x), bf16(gate))
    assert np.allclose(out[0], x[0, 2], atol=1e-20 + 1e-12 * np.abs(x).max())


def test_token_order_does_not_matter_and_weights_are_convex():
    g = np.random.default_rng(4)
    x = bf16(g.standard_normal((5, 4, 40)))
    gate = bf16(g.standard_normal(40) * 0.3)
    a = compress_fold(x, gate)
    b = compress_fold(x[:, [3, 1, 0, 2]], gate)
    assert np.allclose(a, b, rtol=1e-13, atol=1e-15)
    xx = _dec(x)
    assert np.all(a <= xx.max(axis=1) + 1e-12) and np.all(a >= xx.min(axis=1) - 1e-12)


def _m_softmax_over_channels(x_bits, g_bits):
    x, gg = _dec(x_bits), _dec(g_bits)
    out = []
    for b in range(x.shape[0]):
        e = np.exp(x[b] * gg)              # per channel instead of per token
        out.append((e / e.sum(axis=0)).sum(axis=0) * 0 + (e * x[b]).sum(axis=0) / e.sum(axis=0))
    return np.array(out)


def _m_unnormalised(x_bits, g_bits):
    x, gg = _dec(x_bits), _dec(g_bits)
    return np.array([np.exp(x[b] @ gg) @ x[b] for b in range(x.shape[0])])


def _pins_pass(fn):
    """The worked example and the dominant-score pin, for a candidate rule."""
    x = bf16([[[0, 1], [1, 1], [2, 1], [3, 1]]])
    S = 1 + math.e + math.e ** 2 + math.e ** 3
    want = [(math.e + 2 * math.e ** 2 + 3 * math.e ** 3) / S, 1.0]
    if not np.allclose(fn(x, bf16([1, 0]))[0], want, atol=1e-9):
        return False
    g = np.random.default_rng(3)
    xx = _dec(bf16(g.standard_normal((1, 4, 16))))
    xx[0, 2, 0] = 64.0
    gate = np.zeros(16)
    gate[0] = 1.0
    return np.allclose(fn(bf16(xx), bf16(gate))[0], xx[0, 2], atol=1e-9)


def test_pins_accept_the_oracle():
    assert _pins_pass(compress_fold)


@pytest.mark.parametrize("mutant", [_m_softmax_over_channels, _m_unnormalised])
def test_pins_catch_planted_mistakes(mutant):
    assert not _pins_pass(mutant)
