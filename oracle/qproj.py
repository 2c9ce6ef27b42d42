"""Indexer query projection (oracle; test infrastructure only).

What is computed (NKI pull request "Add DeepSeek-V4 CSA attention kernels",
"How the algorithm works", steps table row 2: the indexer query is projected
into 128 channels; launch list: the indexer query projection runs as a GEMV
before the scoring launch):

    q[t, h, c] = sum_i x[t, i] * Wq[h * 128 + c, i]      (then rounded to bfloat16)
    w[t, h]    = sum_i x[t, i] * Ww[h, i]                 (kept in float32)

in float64 from the exact bfloat16 inputs.  Readings where the pages are
silent:
  * the projection is a plain linear map of one input vector per token, with no
    bias, normalisation, rotation or quantisation (none is named);
  * the per-head weights w of the indexer score come from a second linear map of
    the same input (the steps table names a per-head weight next to the
    projection; it is optional here);
  * q is stored in bfloat16 (the scorer's operand type), w in float32.
"""

import numpy as np

from .encoding import decode_bf16


def qproj(x_bits, wq_bits, ww_bits=None, heads=None, d=128):
    """float64 (q [T, heads, d], w [T, heads] or None) before any rounding.

    ``x_bits`` [T, d_in], ``wq_bits`` [heads * d, d_in], ``ww_bits`` None or
    [heads, d_in]: bfloat16 patterns (uint16).
    """
    x = decode_bf16(x_bits)
    wq = decode_bf16(wq_bits)
    T, d_in = x.shape
    if wq.shape[1] != d_in or wq.shape[0] % d:
        raise ValueError("shape mismatch")
    H = wq.shape[0] // d if heads is None else int(heads)
    q = np.zeros((T, H * d), dtype=np.float64)
    for t in range(T):                       # one dot product per output, row by row
        q[t] = wq @ x[t]
    w = None
    if ww_bits is not None:
        ww = decode_bf16(ww_bits)
        if ww.shape != (H, d_in):
            raise ValueError("shape mismatch")
        w = np.stack([ww @ x[t] for t in range(T)])
    return q.reshape(T, H, d), w


def round_bf16(v):
    """Round float64 values to the nearest bfloat16 (ties to even), as float64.

    The neighbours are the two multiples of the quantum around the value: the
    quantum is 2^(e - 7) for a value in [2^e, 2^(e+1)) (8 significant bits), and
    2^-133 below 2^-126, where bfloat16 (binary32's exponent range) is subnormal.
    A result of magnitude 2^128 or more is past the largest finite bfloat16,
    (2 - 2^-7) * 2^127, and becomes infinity; a zero result keeps the sign.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.empty_like(v)
    flat, res = v.ravel(), out.ravel()
    for i, a in enumerate(flat):
        if a == 0 or not np.isfinite(a):
            res[i] = a
            continue
        e = np.floor(np.log2(abs(a)))
        if abs(a) < 2.0 ** e:                     # log2 rounded up just below a power of two
            e -= 1
        e = max(e, -126.0)                        # the subnormal range's fixed quantum
        ulp = 2.0 ** (e - 7)                      # bfloat16 keeps 8 significant bits
        lo = np.floor(a / ulp) * ulp
        hi = lo + ulp
        if a - lo < hi - a:
            res[i] = lo
        elif a - lo > hi - a:
            res[i] = hi
        else:                                     # a tie: the even significand
            res[i] = lo if int(round(lo / ulp)) % 2 == 0 else hi
        if abs(res[i]) >= 2.0 ** 128:
            res[i] = np.copysign(np.inf, a)
        elif res[i] == 0:
            res[i] = np.copysign(0.0, a)
    return out
