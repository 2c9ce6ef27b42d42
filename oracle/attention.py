"""Sparse multi-query decode attention over selected positions (oracle; test
infrastructure only).

What is computed (NKI pull request "Add DeepSeek-V4 CSA attention kernels",
"How the algorithm works": the attention reads only the highest-scoring
compressed positions plus a local window; steps table row 4 "Concatenate and
attend": gather the selected KV rows, add the sliding window, run the
multi-query attention; "The top-k on the GPSIMD engine", last paragraph: K and
V are the same embedding; "Launching a full block": a sliding-window cache
[B, W, head_dim] and a compressed cache [B, T_c, head_dim]).

For one new token of batch row b, with queries q[b, h, :] of every head h:

    rows(b)  = [ kv[b, idx[b, j], :]  for the slots j with 0 <= idx[b, j] < T ]
             + [ win[b, i, :]         for i < win_len[b] ]
    z[h, r]  = scale * (q[b, h, :] . rows(b)[r])
    m[h]     = max( max_r z[h, r], sink[h] )
    l[h]     = sum_r exp(z[h, r] - m[h]) + exp(sink[h] - m[h])
    out[b,h] = sum_r exp(z[h, r] - m[h]) * rows(b)[r] / l[h]
    lse[b,h] = m[h] + log(l[h])

in float64 from the exact bfloat16 / float32 inputs.  Readings where the pages
are silent:
  * every query head attends to the same gathered rows (multi-query: one KV
    head), and each row serves as both key and value;
  * the selected rows and the window rows form one softmax ("concatenate");
  * a slot whose index is outside [0, T) (the -1 padding of the top-k) adds
    nothing; a repeated index is attended once per slot;
  * the attention sink is one logit per head that joins the softmax
    denominator and carries no value; without it the sink terms are absent;
  * the score scale is an argument (1/sqrt(head_dim) in the workloads);
  * with no attended row and no sink the output is 0 and lse is -inf.
"""

import numpy as np

from .encoding import decode_bf16, decode_f32


def _f64(x):
    a = np.asarray(x)
    if a.dtype == np.uint16:
        return decode_bf16(a)
    if a.dtype == np.float32:
        return decode_f32(a)
    return a.astype(np.float64)


def gather_rows(kv, idx_row, win_row, wl):
    """The rows attended by one batch row, in slot order: the valid selected
    cache rows, then the first ``wl`` window rows.  float64 [n, d]."""
    T = kv.shape[0]
    sel = [int(i) for i in idx_row if 0 <= int(i) < T]
    parts = [kv[sel]] if sel else []
    if win_row is not None and wl > 0:
        parts.append(win_row[:wl])
    if not parts:
        return np.zeros((0, kv.shape[1]), dtype=np.float64)
    return np.concatenate(parts, axis=0)


def sparse_attention(q, kv, idx, scale, win=None, win_len=None, sink=None, kv_shared=None):
    """float64 (out [B, H, d], lse [B, H]).

    ``q``    [B, H, d]      bfloat16 patterns (uint16) or floats;
    ``kv``   [T, d] (one cache shared by every batch row) or [B, T, d];
    ``idx``  [B, k] integer slots; entries outside [0, T) are skipped;
    ``win``  None or [B, W, d]; ``win_len`` None (= W) or [B];
    ``sink`` None or [H] float logits;  ``scale`` the score factor.
    ``kv_shared`` forces the reading of a 2-D ``kv`` (default: by its rank).
    """
    qf = _f64(q)
    kvf = _f64(kv)
    B, H, d = qf.shape
    shared = (kvf.ndim == 2) if kv_shared is None else bool(kv_shared)
    winf = None if win is None else _f64(win)
    W = 0 if winf is None else winf.shape[1]
    sk = None if sink is None else _f64(sink).reshape(H)
    idx = np.asarray(idx)
    out = np.zeros((B, H, d), dtype=np.float64)
    lse = np.full((B, H), -np.inf, dtype=np.float64)
    for b in range(B):
        cache = kvf if shared else kvf[b]
        wl = W if win_len is None else max(0, min(int(win_len[b]), W))
        rows = gather_rows(cache, idx[b], None if winf is None else winf[b], wl)
        z = float(scale) * (qf[b] @ rows.T)              # [H, n]
        for h in range(H):
            zh = z[h]
            cand = list(zh)
            if sk is not None:
                cand.append(sk[h])
            if not cand:
                continue                                 # nothing attended: 0, -inf
            m = max(cand)
            e = np.exp(zh - m)
            l = e.sum() + (np.exp(sk[h] - m) if sk is not None else 0.0)
            out[b, h] = (e @ rows) / l
            lse[b, h] = m + np.log(l)
    return out, lse
