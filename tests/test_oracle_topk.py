"""Pins for the top-k oracle and its decoders (CPU only).

The oracle is checked against things other than itself: a brute-force
repeated-maximum selection, an exhaustive sweep of small ternary rows,
hand-worked examples under tests/golden, a library decoder and a library sort
of the values (which is tie-independent), and the invariants every correct
selection satisfies.  The last tests plant mistakes in copies of the oracle and
check that these pins catch them.
"""

import json
import math
import os

import numpy as np
import pytest

from oracle import decode_bf16, decode_f32, topk_rows, topk_row
from oracle.encoding import NEG_INF_BF16, NEG_INF_F32
from sparse_attention_top_ds_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers

def greater(a, b):
    """a ranks strictly above b (NaN above everything, NaNs equal, -0 == +0)."""
    if math.isnan(a):
        return not math.isnan(b)
    if math.isnan(b):
        return False
    return a > b


def brute_topk(values, k, L):
    """Repeatedly take the strict maximum (lowest index wins ties) and remove it."""
    remaining = list(range(L))
    out = []
    for _ in range(min(k, L)):
        best = remaining[0]
        for i in remaining[1:]:
            if greater(values[i], values[best]):
                best = i
        out.append(best)
        remaining.remove(best)
    return out + [-1] * (k - len(out))


def check_invariants(values, sel, k, L):
    """Properties any correct top-k (ties to lower index) must have."""
    m = min(k, L)
    chosen = [int(i) for i in sel if i >= 0]
    assert len(chosen) == m
    assert len(set(chosen)) == m
    assert all(0 <= i < L for i in chosen)
    assert all(i == -1 for i in sel[m:])
    if m == 0 or m == L:
        return
    rest = sorted(set(range(L)) - set(chosen))
    worst = chosen[0]
    for i in chosen:
        if greater(values[worst], values[i]):
            worst = i
    vk = values[worst]
    # every selected value >= every unselected value
    for j in rest:
        assert not greater(values[j], vk)
    # ties with the k-th value: the selected ones are the lowest-index ones
    tied_sel = sorted(i for i in chosen if not greater(values[i], vk) and not greater(vk, values[i]))
    tied_rest = [j for j in rest if not greater(values[j], vk) and not greater(vk, values[j])]
    if tied_rest:
        assert max(tied_sel) < min(tied_rest)


def parse_value(v):
    return float(v) if isinstance(v, str) else float(v)


# ---------------------------------------------------------------- decoders

def test_decode_bf16_every_pattern_matches_library_widening():
    bits = np.arange(65536, dtype=np.uint32)
    lib = (bits << 16).view(np.float32).astype(np.float64)
    mine = decode_bf16(bits)
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], lib[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(mine[~nan]), np.signbit(lib[~nan]))


def test_decode_bf16_known_constants():
    table = {
        0x3F80: 1.0, 0xC000: -2.0, 0x0000: 0.0, 0x4049: 3.140625,
        0x0001: 2.0 ** -133, 0x0080: 2.0 ** -126,
        0x7F7F: (2.0 - 2.0 ** -7) * 2.0 ** 127,
        0x7F80: math.inf, 0xFF80: -math.inf,
    }
    for b, v in table.items():
        assert decode_bf16(np.array([b]))[0] == v, hex(b)
    neg0 = decode_bf16(np.array([0x8000]))[0]
    assert neg0 == 0.0 and math.copysign(1.0, neg0) == -1.0
    assert math.isnan(decode_bf16(np.array([0x7FC0]))[0])


def test_decode_f32_random_patterns_match_library():
    g = np.random.default_rng(5)
    bits = g.integers(0, 2 ** 32, size=200000, dtype=np.uint64).astype(np.uint32)
    lib = bits.view(np.float32).astype(np.float64)
    mine = decode_f32(bits)
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], lib[~nan])
    assert decode_f32(np.array([0x00000001], dtype=np.uint32))[0] == 2.0 ** -149
    assert decode_f32(np.array([0x7F7FFFFF], dtype=np.uint32))[0] == (2 - 2.0 ** -23) * 2.0 ** 127


# ---------------------------------------------------------------- worked examples

def _golden_cases():
    with open(os.path.join(GOLDEN, "topk_worked_examples.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_worked_examples(case, dtype):
    vals = np.array([parse_value(v) for v in case["values"]], dtype=np.float32)
    bits = inputs.f32_to_bf16_bits(vals) if dtype == "bf16" else vals.view(np.uint32)
    if dtype == "bf16":
        # the fixture values are exact in bfloat16; NaN patterns stay NaN
        assert np.array_equal(np.isnan(decode_bf16(bits)), np.isnan(vals))
    k = case["k"]
    vl = None if case["valid_len"] is None else np.array([case["valid_len"]])
    for sorted_index in (False, True):
        idx, val = topk_rows(bits[None, :], dtype, k, vl, sorted_index=sorted_index)
        expect = case["expect"]
        m = sum(1 for e in expect if e >= 0)
        assert sorted(int(i) for i in idx[0, :m]) == sorted(e for e in expect if e >= 0)
        assert list(idx[0, m:]) == [-1] * (k - m)
        if sorted_index:
            assert list(idx[0, :m]) == sorted(idx[0, :m])
        pad = NEG_INF_BF16 if dtype == "bf16" else NEG_INF_F32
        assert all(int(v) == pad for v in val[0, m:])
        assert np.array_equal(val[0, :m], bits[idx[0, :m]])


# ---------------------------------------------------------------- brute force

def test_brute_force_tiny_rows_with_ties():
    g = np.random.default_rng(11)
    pool = np.array([-2.0, -0.0, 0.0, 0.5, 1.0, 1.0, 3.0, np.inf, -np.inf, np.nan])
    for trial in range(400):
        n = int(g.integers(1, 65))
        vals = g.choice(pool[: 7 if trial % 3 else 10], size=n)
        for k in sorted(set([1, n, int(g.integers(1, n + 1)), int(g.integers(1, n + 1))])):
            L = n if trial % 2 else int(g.integers(0, n + 1))
            got = topk_row(vals, k, L)
            assert list(got) == brute_topk(list(vals), k, L), (vals, k, L)


def test_exhaustive_ternary_rows():
    n = 7
    for code in range(3 ** n):
        vals, c = [], code
        for _ in range(n):
            vals.append(float(c % 3))
            c //= 3
        for k in range(1, n + 1):
            assert list(topk_row(np.array(vals), k, n)) == brute_topk(vals, k, n)


# ---------------------------------------------------------------- invariants and library pins

def test_invariants_sampling_like_rows():
    x, planted = inputs.sampling(seed=77, batch=3, n=5000, outliers=20)
    for k in (1, 19, 20, 21, 64, 1024):
        idx, val = topk_rows(x, "f32", k)
        for t in range(3):
            check_invariants(list(x[t].astype(np.float64)), list(idx[t]), k, 5000)
            if k >= 20:
                assert set(planted[t]).issubset(set(idx[t]))
            # the multiset of selected values is tie-independent: library sort
            lib = np.sort(x[t].astype(np.float64))[::-1][:k]
            assert np.array_equal(np.sort(val[t].view(np.float32).astype(np.float64))[::-1], lib)


def test_invariants_bf16_rows_with_many_ties():
    bits = inputs.standalone(seed=3, batch=2, n=8192)
    dec = decode_bf16(bits)
    assert len(np.unique(dec[0])) < 2000          # bfloat16 N(0,1): heavy ties
    vl = np.array([8192, 5000])
    for k in (1, 512, 2048, 8192):
        idx, val = topk_rows(bits, "bf16", k, vl)
        for t in range(2):
            check_invariants(list(dec[t]), list(idx[t]), k, int(vl[t]))
            m = min(k, int(vl[t]))
            lib = np.sort(dec[t, : vl[t]])[::-1][:m]
            assert np.array_equal(np.sort(decode_bf16(val[t, :m]))[::-1], lib)


def test_ascending_rows_pick_the_tail():
    bits = inputs.sort_rows_ascending_bf16(inputs.standalone(seed=4, batch=1, n=4096))
    dec = decode_bf16(bits[0])
    assert np.all(np.diff(dec) >= 0)
    idx, _ = topk_rows(bits, "bf16", 100)
    # ascending values: the selection is the last 100 positions, except that
    # values equal to the 100th-largest are taken from the lowest index first
    vk = np.sort(dec)[::-1][99]
    above = set(np.nonzero(dec > vk)[0])
    ties = list(np.nonzero(dec == vk)[0])
    expect = above | set(ties[: 100 - len(above)])
    assert set(idx[0]) == expect


def test_sorted_index_option_same_set_ascending():
    x, _ = inputs.sampling(seed=9, batch=2, n=3000)
    a, va = topk_rows(x, "f32", 300)
    b, vb = topk_rows(x, "f32", 300, sorted_index=True)
    for t in range(2):
        assert set(a[t]) == set(b[t])
        assert np.all(np.diff(b[t]) > 0)
        assert np.array_equal(vb[t], x[t].view(np.uint32)[b[t]])


# ---------------------------------------------------------------- planted mistakes

def _mutant_high_index_ties(values, k, L):
    v = np.asarray(values, dtype=np.float64)[:L]
    order = np.lexsort((-np.arange(L), -v))          # ties to the HIGHER index
    out = np.full(k, -1)
    out[: min(k, L)] = order[: min(k, L)]
    return out


def _mutant_signed_zero(values, k, L):
    v = np.asarray(values, dtype=np.float64)[:L]
    key = np.where(v == 0, np.where(np.signbit(v), -1e-300, 1e-300), v)   # -0 < +0
    order = np.lexsort((np.arange(L), -key))
    out = np.full(k, -1)
    out[: min(k, L)] = order[: min(k, L)]
    return out


def _mutant_valid_len_off_by_one(values, k, L):
    return topk_row(values, k, min(L + 1, len(values)))


@pytest.mark.parametrize("mutant", [_mutant_high_index_ties, _mutant_signed_zero,
                                    _mutant_valid_len_off_by_one])
def test_pins_catch_planted_mistakes(mutant):
    caught = False
    for case in _golden_cases():
        vals = np.array([parse_value(v) for v in case["values"]])
        L = len(vals) if case["valid_len"] is None else case["valid_len"]
        got = sorted(int(i) for i in mutant(vals, case["k"], L) if i >= 0)
        if got != sorted(e for e in case["expect"] if e >= 0):
            caught = True
    g = np.random.default_rng(1)
    for _ in range(50):
        vals = g.choice([0.0, -0.0, 1.0, 2.0], size=12)
        L = int(g.integers(0, 12))
        if list(mutant(vals, 4, L)) != brute_topk(list(vals), 4, L):
            caught = True
    assert caught
