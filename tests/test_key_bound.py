"""The stash top-k's stream tests each score with one float compare against
the threshold key's value (topk_kernel.cuh: F32Keys/BF16Keys::bound and ::ge)
instead of converting the score to its order-preserving key.  This checks, on
the CPU, the equivalence the kernel relies on: for every score x and key
threshold t, key(x) >= t holds exactly when !(x < bound(t)) -- or, where
bound(t) is a NaN (t above key(+inf) or below key(-inf)), the float test lets
every score through, a superset that never drops a key >= t.

key() is restated from the library's documented order: larger key = larger
value, -0 folded onto +0, every NaN the top key."""

import numpy as np


def key32(b):
    b = b.astype(np.uint32)
    nan = (b & 0x7FFFFFFF) > 0x7F800000
    b = np.where(b == 0x80000000, np.uint32(0), b)
    k = np.where(b & 0x80000000, ~b, b | np.uint32(0x80000000)).astype(np.uint32)
    return np.where(nan, np.uint32(0xFFFFFFFF), k)


def bound32(t):
    t = np.uint32(t)
    bits = (t & np.uint32(0x7FFFFFFF)) if (t & np.uint32(0x80000000)) else ~t
    return np.array([bits], dtype=np.uint32).view(np.float32)[0]


def key16(b):
    b = b.astype(np.uint32) & 0xFFFF
    nan = (b & 0x7FFF) > 0x7F80
    b = np.where(b == 0x8000, np.uint32(0), b)
    k = np.where(b & 0x8000, (~b) & 0xFFFF, b | 0x8000).astype(np.uint32)
    return np.where(nan, np.uint32(0xFFFF), k)


def bound16(t):
    t = int(t)
    bits = (t & 0x7FFF) if (t & 0x8000) else ((~t) & 0xFFFF)
    return np.array([bits << 16], dtype=np.uint32).view(np.float32)[0]


def _check(keys, xs_float, t, bound):
    want = keys >= t
    with np.errstate(invalid="ignore"):
        got = ~(xs_float < bound(t))
    bf = bound(t)
    if np.isnan(bf):
        assert np.all(got), f"t={t:#x}: a NaN bound must pass every score"
    else:
        assert np.array_equal(got, want), f"t={t:#x}: float test differs from key test"


def test_bfloat16_every_score_against_many_thresholds():
    raw = np.arange(65536, dtype=np.uint32)
    keys = key16(raw)
    xs = (raw << 16).view(np.float32)
    for t in list(range(0, 65536, 97)) + [0, 1, 0x007F, 0x0080, 0x7FFF, 0x8000, 0x8001, 0xFF80, 0xFF81, 0xFFFF]:
        _check(keys, xs, t, bound16)


def test_float32_scores_with_special_values_against_many_thresholds():
    g = np.random.default_rng(11)
    specials = np.array([0x00000000, 0x80000000, 0x00000001, 0x80000001, 0x007FFFFF, 0x807FFFFF, 0x00800000,
                         0x80800000, 0x7F7FFFFF, 0xFF7FFFFF, 0x7F800000, 0xFF800000, 0x7FC00000, 0xFFC00000,
                         0x7F800001, 0xFFFFFFFF, 0x3F800000, 0xBF800000], dtype=np.uint32)
    raw = np.concatenate([specials, g.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)])
    keys = key32(raw)
    xs = raw.view(np.float32)
    ts = np.concatenate([key32(specials), key32(specials) + 1, key32(specials) - 1,
                         g.integers(0, 2 ** 32, size=3000, dtype=np.uint64).astype(np.uint32),
                         np.arange(0, 4096, dtype=np.uint32) << 20])  # every 12-bit bin edge
    for t in np.unique(ts.astype(np.uint32)):
        _check(keys, xs, int(t), bound32)
