"""Pins for the sparse-attention oracle (CPU only).

Checked against a library routine (torch's scaled_dot_product_attention in
float64 when every cache row is selected), closed forms (identical rows, zero
queries, a two-row case worked by hand, a repeated slot, the sink's share, empty
inputs) and invariants (slot order, skipped slots, moving a row between the cache and the
window, per-batch caches, the scale folded into q, convexity).  Mutated copies
of the attention rule are shown to fail the pins.
"""

import math

import numpy as np
import pytest
import torch

from oracle import sparse_attention
from oracle.attention import gather_rows
from sparse_attention_top_ds_b200 import inputs


def bf16(a):
    return inputs.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _case(seed, B=2, H=6, d=16, T=40, k=12, W=5, with_sink=True):
    g = np.random.default_rng(seed)
    q = bf16(g.standard_normal((B, H, d)))
    kv = bf16(g.standard_normal((T, d)))
    win = bf16(g.standard_normal((B, W, d)))
    idx = np.stack([g.choice(T, size=k, replace=False) for _ in range(B)]).astype(np.int32)
    sink = g.standard_normal(H).astype(np.float32) if with_sink else None
    return q, kv, win, idx, sink


def _dec(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- library routine

@pytest.mark.parametrize("scale", [1.0 / 4.0, 0.37])
def test_all_rows_selected_equals_torch_sdpa(scale):
    B, H, d, T = 3, 5, 16, 23
    g = np.random.default_rng(7)
    q = bf16(g.standard_normal((B, H, d)))
    kv = bf16(g.standard_normal((T, d)))
    idx = np.stack([g.permutation(T) for _ in range(B)])
    out, _ = sparse_attention(q, kv, idx, scale)
    qt = torch.from_numpy(_dec(q)).unsqueeze(2)                  # [B, H, 1, d]
    kt = torch.from_numpy(_dec(kv)).expand(B, H, T, d)           # one KV head for all query heads
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, scale=scale).squeeze(2).numpy()
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-14)


def test_window_only_equals_torch_sdpa():
    B, H, d, W = 2, 4, 8, 9
    g = np.random.default_rng(8)
    q = bf16(g.standard_normal((B, H, d)))
    kv = bf16(g.standard_normal((3, d)))
    win = bf16(g.standard_normal((B, W, d)))
    idx = np.full((B, 4), -1, dtype=np.int32)
    out, _ = sparse_attention(q, kv, idx, 0.5, win=win)
    for b in range(B):
        qt = torch.from_numpy(_dec(q[b])).view(1, H, 1, d)
        kt = torch.from_numpy(_dec(win[b])).view(1, 1, W, d).expand(1, H, W, d)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, scale=0.5).view(H, d).numpy()
        assert np.allclose(out[b], ref, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- closed forms

def test_two_rows_worked_by_hand():
    # q = (2, 0), rows (1, 0) and (0, 1), scale 1/2: the scores are 1 and 0,
    # the weights e/(e+1) and 1/(e+1), so out = (sigmoid(1), sigmoid(-1)) and
    # lse = log(1 + e).
    q = bf16([[[2.0, 0.0]]])
    kv = bf16([[1.0, 0.0], [0.0, 1.0], [5.0, 5.0]])
    out, lse = sparse_attention(q, kv, np.array([[1, 0, -1]]), 0.5)
    assert out[0, 0, 0] == pytest.approx(0.7310585786300049, abs=1e-15)
    assert out[0, 0, 1] == pytest.approx(0.2689414213699951, abs=1e-15)
    assert lse[0, 0] == pytest.approx(1.3132616875182228, abs=1e-15)


def test_identical_rows_return_the_row():
    d, n = 16, 9
    g = np.random.default_rng(9)
    v = bf16(g.standard_normal(d))
    kv = np.tile(v, (n, 1))
    q = bf16(g.standard_normal((1, 3, d)))
    out, lse = sparse_attention(q, kv, np.arange(n)[None], 0.3)
    assert np.allclose(out[0], np.tile(_dec(v), (3, 1)), rtol=1e-14, atol=0)
    z = 0.3 * (_dec(q[0]) @ _dec(v))
    assert np.allclose(lse[0], z + math.log(n), rtol=1e-13, atol=1e-13)


def test_identical_rows_with_sink_closed_form():
    # n equal rows with score z and a sink s: out = v * n e^z / (n e^z + e^s).
    d, n = 8, 6
    g = np.random.default_rng(10)
    v = bf16(g.standard_normal(d))
    kv = np.tile(v, (n, 1))
    q = bf16(g.standard_normal((1, 2, d)))
    sink = np.array([0.5, -3.0], dtype=np.float32)
    out, lse = sparse_attention(q, kv, np.arange(n)[None], 0.25, sink=sink)
    for h in range(2):
        z = 0.25 * float(_dec(q[0, h]) @ _dec(v))
        s = float(sink[h])
        share = n * math.exp(z) / (n * math.exp(z) + math.exp(s))
        assert np.allclose(out[0, h], share * _dec(v), rtol=1e-13, atol=1e-15)
        assert lse[0, h] == pytest.approx(math.log(n * math.exp(z) + math.exp(s)), rel=1e-13)


def test_zero_queries_average_the_rows():
    B, H, d, T, k, W = 2, 3, 8, 30, 7, 4
    _, kv, win, idx, _ = _case(11, B, H, d, T, k, W)
    q = np.zeros((B, H, d), dtype=np.uint16)
    wl = np.array([4, 1])
    out, lse = sparse_attention(q, kv, idx, 0.7, win=win, win_len=wl)
    for b in range(B):
        rows = np.concatenate([_dec(kv)[idx[b]], _dec(win[b])[:wl[b]]])
        assert np.allclose(out[b], np.tile(rows.mean(0), (H, 1)), rtol=1e-13, atol=1e-15)
        assert np.allclose(lse[b], math.log(len(rows)), rtol=1e-14)


def test_sink_of_log_n_halves_the_average():
    # zero queries, n rows and sink log(n): the sink takes half of the mass.
    n, d = 10, 4
    g = np.random.default_rng(12)
    kv = bf16(g.standard_normal((n, d)))
    q = np.zeros((1, 1, d), dtype=np.uint16)
    out, lse = sparse_attention(q, kv, np.arange(n)[None], 1.0, sink=np.array([math.log(n)]))
    assert np.allclose(out[0, 0], _dec(kv).mean(0) / 2, rtol=1e-13, atol=1e-15)
    assert lse[0, 0] == pytest.approx(math.log(2 * n), rel=1e-14)


def test_nothing_attended():
    q = bf16(np.ones((2, 3, 4)))
    kv = bf16(np.ones((5, 4)))
    idx = np.array([[-1, 5, 99], [-7, -1, -1]])
    win = bf16(np.ones((2, 3, 4)))
    out, lse = sparse_attention(q, kv, idx, 1.0, win=win, win_len=[0, -2])
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    sink = np.array([1.5, -2.0, 0.0], dtype=np.float32)
    out, lse = sparse_attention(q, kv, idx, 1.0, win=win, win_len=[0, 0], sink=sink)
    assert np.all(out == 0) and np.allclose(lse, np.tile(sink.astype(np.float64), (2, 1)))


# ---------------------------------------------------------------- invariants

def test_slot_order_does_not_matter():
    q, kv, win, idx, sink = _case(13)
    a = sparse_attention(q, kv, idx, 0.25, win=win, sink=sink)
    g = np.random.default_rng(0)
    idx2 = np.stack([g.permutation(r) for r in idx])
    win2 = np.stack([w[g.permutation(w.shape[0])] for w in win])
    b = sparse_attention(q, kv, idx2, 0.25, win=win2, sink=sink)
    assert np.allclose(a[0], b[0], rtol=1e-12, atol=1e-15) and np.allclose(a[1], b[1], rtol=1e-13)


def test_out_of_range_slots_are_skipped():
    q, kv, win, idx, sink = _case(14, T=40)
    a = sparse_attention(q, kv, idx, 0.25, win=win, sink=sink)
    pad = np.tile(np.array([-1, 40, 41, -100, 1 << 30]), (idx.shape[0], 1))
    b = sparse_attention(q, kv, np.concatenate([pad[:, :2], idx, pad[:, 2:]], 1), 0.25, win=win, sink=sink)
    assert np.allclose(a[0], b[0], rtol=1e-13, atol=1e-15) and np.allclose(a[1], b[1], rtol=1e-14)


def test_a_row_may_move_between_cache_and_window():
    # Selecting cache row r is the same as offering r's values in the window.
    q, kv, win, idx, sink = _case(15, B=2, W=5)
    wl = np.array([3, 2])
    a = sparse_attention(q, kv, idx, 0.25, win=win, win_len=wl, sink=sink)
    idx2 = idx.copy()
    win2 = win.copy()
    for b in range(2):
        win2[b, wl[b]] = kv[idx[b, 0]]
        idx2[b, 0] = -1
    b_ = sparse_attention(q, kv, idx2, 0.25, win=win2, win_len=wl + 1, sink=sink)
    assert np.allclose(a[0], b_[0], rtol=1e-12, atol=1e-15) and np.allclose(a[1], b_[1], rtol=1e-13)


def test_per_batch_caches_are_independent():
    B, H, d, T = 3, 2, 8, 20
    g = np.random.default_rng(16)
    q = bf16(g.standard_normal((B, H, d)))
    kv3 = bf16(g.standard_normal((B, T, d)))
    idx = np.stack([g.choice(T, 6, replace=False) for _ in range(B)])
    out, lse = sparse_attention(q, kv3, idx, 0.5)
    for b in range(B):
        o1, l1 = sparse_attention(q[b:b + 1], kv3[b], idx[b:b + 1], 0.5)
        assert np.allclose(out[b], o1[0], rtol=1e-14, atol=0) and np.allclose(lse[b], l1[0], rtol=1e-14)


def test_scale_folds_into_the_queries():
    q, kv, win, idx, sink = _case(17)
    a = sparse_attention(q, kv, idx, 0.5, win=win, sink=sink)
    q2 = (_dec(q) * 2.0)
    b = sparse_attention(q2, kv, idx, 0.25, win=win, sink=sink)
    assert np.allclose(a[0], b[0], rtol=1e-13, atol=1e-15) and np.allclose(a[1], b[1], rtol=1e-14)


def test_repeated_slot_counts_once_per_slot():
    # slots [0, 0, 1] with z = (1, 1, 0): row 0 carries weight 2e / (2e + 1)
    q = bf16([[[2.0, 0.0]]])
    kv = bf16([[1.0, 0.0], [0.0, 1.0]])
    out, lse = sparse_attention(q, kv, np.array([[0, 0, 1]]), 0.5)
    e2 = 2.0 * math.e
    assert abs(out[0, 0, 0] - e2 / (e2 + 1.0)) < 1e-15
    assert abs(out[0, 0, 1] - 1.0 / (e2 + 1.0)) < 1e-15
    assert abs(lse[0, 0] - math.log(e2 + 1.0)) < 1e-14


def test_repeated_slot_equals_the_row_also_in_the_window():
    q, kv, win, idx, sink = _case(20, W=3)
    rep = idx.copy()
    rep[:, -1] = rep[:, 0]                       # the last slot repeats the first
    w2 = win.copy()
    for b in range(q.shape[0]):
        w2[b, 0] = kv[idx[b, 0]]                 # the same row as the window's only row
    a = sparse_attention(q, kv, rep, 0.3, win=win, win_len=np.zeros(2, np.int32), sink=sink)
    c = sparse_attention(q, kv, idx[:, :-1], 0.3, win=w2,
                         win_len=np.ones(2, np.int32), sink=sink)
    assert np.allclose(a[0], c[0], atol=1e-13) and np.allclose(a[1], c[1], atol=1e-13)


def test_output_is_inside_the_rows_hull():
    q, kv, win, idx, _ = _case(18, with_sink=False)
    out, _ = sparse_attention(q, kv, idx, 2.0, win=win)
    for b in range(q.shape[0]):
        rows = gather_rows(_dec(kv), idx[b], _dec(win[b]), win.shape[1])
        assert np.all(out[b] <= rows.max(0) + 1e-12) and np.all(out[b] >= rows.min(0) - 1e-12)


# ---------------------------------------------------------------- planted mistakes

def _pins_pass(fn):
    """True if the candidate rule passes the worked example, the sink closed
    form and the window/cache move."""
    q = bf16([[[2.0, 0.0]]])
    kv = bf16([[1.0, 0.0], [0.0, 1.0]])
    o, l = fn(q, kv, np.array([[1, 0]]), 0.5, None, None, None)
    if not (abs(o[0, 0, 0] - 0.7310585786300049) < 1e-12 and abs(l[0, 0] - 1.3132616875182228) < 1e-12):
        return False
    o, l = fn(q, kv, np.array([[0, 0, 1]]), 0.5, None, None, None)
    if abs(o[0, 0, 0] - 2 * math.e / (2 * math.e + 1)) > 1e-12:
        return False
    o, l = fn(np.zeros((1, 1, 2), np.uint16), kv, np.array([[0, 1]]), 1.0, None, None, np.array([math.log(2)]))
    if not np.allclose(o[0, 0], _dec(kv).mean(0) / 2, atol=1e-12):
        return False
    q3, kv3, win3, idx3, sink3 = _case(19, B=2, W=4)
    a = fn(q3, kv3, idx3, 0.25, win3, np.array([2, 3]), sink3)
    i2, w2 = idx3.copy(), win3.copy()
    for b, wl in enumerate([2, 3]):
        w2[b, wl] = kv3[idx3[b, 0]]
        i2[b, 0] = -1
    c = fn(q3, kv3, i2, 0.25, w2, np.array([3, 4]), sink3)
    return np.allclose(a[0], c[0], atol=1e-12)


def _correct(q, kv, idx, scale, win, wl, sink):
    return sparse_attention(q, kv, idx, scale, win=win, win_len=wl, sink=sink)


def _m_sink_carries_value(q, kv, idx, scale, win, wl, sink):
    out, lse = sparse_attention(q, kv, idx, scale, win=win, win_len=wl, sink=sink)
    if sink is None:
        return out, lse
    # the sink's share redistributed over the rows (as if the sink were absent)
    out2, _ = sparse_attention(q, kv, idx, scale, win=win, win_len=wl, sink=None)
    return out2, lse


def _m_separate_softmax(q, kv, idx, scale, win, wl, sink):
    # window rows and selected rows normalised separately, then averaged
    if win is None:
        return sparse_attention(q, kv, idx, scale, sink=sink)
    a = sparse_attention(q, kv, idx, scale, sink=sink)
    b = sparse_attention(q, kv, np.full_like(idx, -1), scale, win=win, win_len=wl, sink=sink)
    return (a[0] + b[0]) / 2, np.logaddexp(a[1], b[1])


def _m_window_of_batch0(q, kv, idx, scale, win, wl, sink):
    if win is None:
        return sparse_attention(q, kv, idx, scale, sink=sink)
    w0 = np.repeat(win[:1], win.shape[0], 0)
    return sparse_attention(q, kv, idx, scale, win=w0, win_len=wl, sink=sink)


def _m_sqrt_scale(q, kv, idx, scale, win, wl, sink):
    return sparse_attention(q, kv, idx, math.sqrt(scale), win=win, win_len=wl, sink=sink)


def _m_dedup_slots(q, kv, idx, scale, win, wl, sink):
    # a row selected by several slots attended once
    d = np.array(idx).copy()
    for b in range(d.shape[0]):
        seen = set()
        for j in range(d.shape[1]):
            if int(d[b, j]) in seen:
                d[b, j] = -1
            seen.add(int(d[b, j]))
    return sparse_attention(q, kv, d, scale, win=win, win_len=wl, sink=sink)


def test_pins_accept_the_oracle():
    assert _pins_pass(_correct)


@pytest.mark.parametrize("mutant", [_m_sink_carries_value, _m_separate_softmax, _m_window_of_batch0,
                                    _m_sqrt_scale, _m_dedup_slots])
def test_pins_catch_planted_mistakes(mutant):
    assert not _pins_pass(mutant)
