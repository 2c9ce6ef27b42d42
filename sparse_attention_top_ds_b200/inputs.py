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
* ``qproj``           the indexer query projection of a decode step: 8 token
                      rows of width 1536, Wq [64 x 128, 1536] ~ N(0, 1/(128 * 1536))
                      (so q ~ N(0, 1/128), the indexer configs' query scale) and
                      Ww [64, 1536] ~ N(0, 1/1536).
* ``attention``       sparse-attention decode: 8 new tokens x 128 query heads x
                      head_dim 512, one compressed KV cache of 32768 rows per
                      batch row, k = 1024 selected rows drawn below a valid
                      length ~ U{4096..32768}, a window of 128 rows, and one
                      sink logit per head; values ~ N(0, 1).

bfloat16 values are produced by drawing float32 samples and rounding them to
the nearest bfloat16, ties to even, and are returned as uint16 bit patterns.
"""

import numpy as np

SEED_STANDALONE = 1001
SEED_SAMPLING = 1002
SEED_INDEXER = 1003
SEED_DECODE = 1004
SEED_PREFILL = 1005
SEED_ATTENTION = 1006
SEED_QPROJ = 1007
SEED_COMPRESS = 1008


def rng(seed):
    return np.random.default_rng(seed)


def f32_to_bf16_bits(x):
    """Round float32 values to the nearest bfloat16 (ties to even); uint16 patterns.

    Only finite inputs are expected (the generators draw no NaN).
    """
    u = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32)
    # for finite values u + 0x8000 stays below 2^32, so uint32 arithmetic is exact
    out = (u >> np.uint32(16)) & np.uint32(1)
    out += np.uint32(0x7FFF)
    out += u
    out >>= np.uint32(16)
    return out.astype(np.uint16)


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


def attention(seed=SEED_ATTENTION, batch=8, heads=128, d=512, T=32768, k=1024, W=128, shared_cache=False,
              vl_lo=4096, vl_hi=32768, sink=True, holes=0.0, win_len=None):
    """Sparse-attention decode inputs.

    Returns a dict: q [batch, heads, d], kv [T, d] (``shared_cache``) or
    [batch, T, d], win [batch, W, d] (bfloat16 patterns of N(0, 1) samples);
    idx int32 [batch, k]: distinct rows drawn uniformly below a valid length
    ~ U{vl_lo..vl_hi} (capped at T), -1 in the slots past that length; a
    fraction ``holes`` of the slots is then replaced by -1 or by rows at or
    past T (skipped slots); win_len int32 [batch] (given, or W); sink float32
    [heads] ~ N(0, 1) or None.
    """
    g = rng(seed)
    q = f32_to_bf16_bits(g.standard_normal((batch, heads, d), dtype=np.float32))
    shape = (T, d) if shared_cache else (batch, T, d)
    kv = f32_to_bf16_bits(g.standard_normal(shape, dtype=np.float32))
    win = f32_to_bf16_bits(g.standard_normal((batch, W, d), dtype=np.float32))
    idx = np.full((batch, k), -1, dtype=np.int32)
    for b in range(batch):
        L = int(min(T, g.integers(min(vl_lo, T), min(vl_hi, T), endpoint=True)))
        m = min(k, L)
        idx[b, :m] = g.choice(L, size=m, replace=False)
    if holes > 0 and k > 0:
        hit = g.random((batch, k)) < holes
        bad = np.where(g.random((batch, k)) < 0.5, -1, T + g.integers(0, 1000, size=(batch, k)))
        idx = np.where(hit, bad, idx).astype(np.int32)
    wl = np.full(batch, W, dtype=np.int32) if win_len is None else np.asarray(win_len, dtype=np.int32)
    sk = g.standard_normal(heads).astype(np.float32) if sink else None
    return dict(q=q, kv=kv, win=win, idx=idx, win_len=wl, sink=sk)


def qproj(seed=SEED_QPROJ, T=8, d_in=1536, heads=64, d=128, with_w=True):
    """Projection inputs: (x [T, d_in], wq [heads * d, d_in], ww [heads, d_in] or None),
    bfloat16 patterns of x ~ N(0, 1), wq ~ N(0, 1/(d * d_in)), ww ~ N(0, 1/d_in)."""
    g = rng(seed)
    x = f32_to_bf16_bits(g.standard_normal((T, d_in), dtype=np.float32))
    wq = f32_to_bf16_bits(g.standard_normal((heads * d, d_in), dtype=np.float32) * np.float32(1.0 / np.sqrt(d * d_in)))
    ww = None
    if with_w:
        ww = f32_to_bf16_bits(g.standard_normal((heads, d_in), dtype=np.float32) * np.float32(1.0 / np.sqrt(d_in)))
    return x, wq, ww


def attention_slots(seed, batch=8, T=32768, k=1024, vl_lo=4096, vl_hi=32768):
    """Another draw of the attention workload's slots alone (int32 [batch, k]),
    with the same rule as ``attention``: distinct rows below a valid length
    ~ U{vl_lo..vl_hi}, -1 past it."""
    g = rng(seed)
    idx = np.full((batch, k), -1, dtype=np.int32)
    for b in range(batch):
        L = int(min(T, g.integers(min(vl_lo, T), min(vl_hi, T), endpoint=True)))
        m = min(k, L)
        idx[b, :m] = g.choice(L, size=m, replace=False)
    return idx


def compress(seed=SEED_COMPRESS, batch=8, D=512, gate_scale=1.0):
    """Compressor inputs: (rows [batch, 4, D], gate [D]) bfloat16 patterns of
    rows ~ N(0, 1) and gate ~ N(0, gate_scale^2 / D) (gate scores ~ N(0, gate_scale^2))."""
    g = rng(seed)
    rows = f32_to_bf16_bits(g.standard_normal((batch, 4, D), dtype=np.float32))
    gate = f32_to_bf16_bits(g.standard_normal(D, dtype=np.float32) * np.float32(gate_scale / np.sqrt(D)))
    return rows, gate
