"""Seeded synthetic inputs for the selection step.

This module is shared by the tests, the benchmark and the oracle's callers.  It
draws random numbers and stores them in the input formats; it holds none of the
selection step's arithmetic (no key transform, no scoring, no selection).

Workloads (sizes and distributions of the selection step's headline cases):

* ``standalone``      4 rows x 8192 bfloat16 scores ~ N(0, 1), k = 512.
* ``sampling``        64 rows x 129280 float32 logits ~ N(0, 3^2) with 20
                      distinct positions per row set to exactly +15.0.
* ``indexer_factors`` the factors of indexer-style score rows: q [B, 64, 128]
                      and keys [n, 128] bfloat16 ~ N(0, 1/128) (the second
                      argument is the variance), w [B, 64] float32 ~ U(0, 1).
* ``decode``          8 query rows x 64 heads x 128 against one key cache of
                      32768 positions, w ~ U(0, 1), valid_len ~ U{4096..32768}.
* ``prefill``         4096 query rows x 64 heads x 128 against 32768 keys with
                      the causal prefix valid_len[t] = floor((t + c) / 4),
                      c = 4 * (S - T/4).

bfloat16 values are produced by drawing float32 samples and rounding them to
the nearest bfloat16, ties to even, and are returned as uint16 bit patterns.
"""

import numpy as np

SEED_STANDALONE = 1001
SEED_SAMPLING = 1002
SEED_INDEXER = 1003
SEED_DECODE = 1004
SEED_PREFILL = 1005


def rng(seed):
    return np.random.default_rng(seed)


def f32_to_bf16_bits(x):
    """Round float32 values to the nearest bfloat16 (ties to even); uint16 patterns.

    Only finite inputs are expected (the generators draw no NaN).
    """
    u = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((u >> 16) & 1)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits):
    """Widen bfloat16 patterns to float32 (exact: a bfloat16 is a truncated float32)."""
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32)


def standalone(seed=SEED_STANDALONE, batch=4, n=8192):
    """[batch, n] bfloat16 patterns of N(0, 1) samples."""
    g = rng(seed)
    return f32_to_bf16_bits(g.standard_normal((batch, n), dtype=np.float32))


def sampling(seed=SEED_SAMPLING, batch=64, n=129280, outliers=20, outlier_value=15.0):
    """[batch, n] float32 logits ~ N(0, 9) with ``outliers`` planted values per row.

    Returns (logits, planted_positions [batch, outliers]).
    """
    g = rng(seed)
    x = (g.standard_normal((batch, n), dtype=np.float32) * np.float32(3.0)).astype(np.float32)
    planted = np.empty((batch, outliers), dtype=np.int64)
    for t in range(batch):
        pos = g.choice(n, size=outliers, replace=False)
        planted[t] = np.sort(pos)
        x[t, pos] = np.float32(outlier_value)
    return x, planted


def indexer_factors(seed=SEED_INDEXER, batch=8, n=32768, heads=64, d=128):
    """Factors of indexer-style rows: (q [batch,heads,d] u16, keys [n,d] u16, w [batch,heads] f32)."""
    g = rng(seed)
    std = np.float32(1.0 / np.sqrt(128.0))
    q = f32_to_bf16_bits(g.standard_normal((batch, heads, d), dtype=np.float32) * std)
    keys = f32_to_bf16_bits(g.standard_normal((n, d), dtype=np.float32) * std)
    w = g.random((batch, heads), dtype=np.float32)
    return q, keys, w


def sort_rows_ascending_bf16(bits):
    """The adversarial variant: every bfloat16 row rearranged into ascending value order."""
    f = bf16_bits_to_f32(bits)
    s = np.sort(f, axis=1)
    return (np.ascontiguousarray(s).view(np.uint32) >> 16).astype(np.uint16)


def decode(seed=SEED_DECODE, batch=8, heads=64, d=128, S=32768, vl_lo=4096, vl_hi=32768):
    """Decode-step inputs: (q u16 [batch,heads,d], kcache u16 [S,d], w f32 [batch,heads], vl i32 [batch])."""
    g = rng(seed)
    std = np.float32(1.0 / np.sqrt(128.0))
    q = f32_to_bf16_bits(g.standard_normal((batch, heads, d), dtype=np.float32) * std)
    kc = f32_to_bf16_bits(g.standard_normal((S, d), dtype=np.float32) * std)
    w = g.random((batch, heads), dtype=np.float32)
    vl = g.integers(vl_lo, vl_hi, size=batch, endpoint=True).astype(np.int32)
    vl = np.minimum(vl, S).astype(np.int32)
    return q, kc, w, vl


def causal_valid_len(T, S):
    """valid_len[t] = floor((t + c) / 4) with c = 4 * (S - T/4), as int32."""
    c = 4 * (S - T // 4)
    t = np.arange(T, dtype=np.int64)
    return ((t + c) // 4).astype(np.int32)


def prefill(seed=SEED_PREFILL, T=4096, heads=64, d=128, S=32768):
    """Prefill inputs: (q u16 [T,heads,d], kcache u16 [S,d], w f32 [T,heads], vl i32 [T])."""
    g = rng(seed)
    std = np.float32(1.0 / np.sqrt(128.0))
    q = f32_to_bf16_bits(g.standard_normal((T, heads, d), dtype=np.float32) * std)
    kc = f32_to_bf16_bits(g.standard_normal((S, d), dtype=np.float32) * std)
    w = g.random((T, heads), dtype=np.float32)
    return q, kc, w, causal_valid_len(T, S)


def sample_rows(seed, total, count):
    """A seeded, sorted subset of ``count`` distinct row indices out of ``total``."""
    g = rng(seed + 7919)
    return np.sort(g.choice(total, size=min(count, total), replace=False))
