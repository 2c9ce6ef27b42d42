"""Lightning-indexer score and its top-k (oracle; test infrastructure only).

What is computed (NKI pull request "Add DeepSeek-V4 CSA attention kernels",
"How the algorithm works", steps table, row 2 "Lightning indexer": queries and
keys live in 128 indexer channels, and every compressed position is scored with
a multi-query product, a ReLU and a per-head weight; row 3 selects the
highest-scoring positions):

    score[t, s] = sum over heads h of  w[t, h] * max(0, sum over c of q[t,h,c] * k[s,c])

for positions s < valid_len[t], in float64 from the exact bfloat16 / float32
inputs.  Readings where the pages are silent:
  * the ReLU applies to each head's dot product, then the weight multiplies it,
    then the heads are summed (the order the steps table names them in);
  * there is no extra scale factor (any scale folds into w);
  * w is per token and head, of any sign;
  * one key cache [S, d] is shared by every query row, or each row has its own
    [S, d] cache (the [B, T_c, index_head_dim] indexer cache of "Launching a
    full block");
  * positions at or beyond valid_len[t] are not scored and never selected.
"""

import numpy as np

from .encoding import decode_bf16, decode_f32
from .topk import topk_row


def indexer_scores(q_bits, k_bits, w, valid_len=None):
    """float64 score rows.

    ``q_bits`` [batch, heads, d] bfloat16 patterns (uint16);
    ``k_bits`` [S, d] bfloat16 patterns (uint16), one key cache shared by every
               row, or [batch, S, d], one cache per row;
    ``w``      [batch, heads] float32 (or float64) weights;
    ``valid_len`` None or [batch] prefix lengths.
    Returns [batch, S] float64 with NaN at positions s >= valid_len[t]
    (positions that are not scored).
    """
    q = decode_bf16(q_bits)
    kc = decode_bf16(k_bits)
    wa = np.asarray(w)
    w64 = decode_f32(wa) if wa.dtype == np.float32 else wa.astype(np.float64)
    batch, heads, d = q.shape
    per_row = kc.ndim == 3
    S = kc.shape[-2]
    if kc.shape[-1] != d or w64.shape != (batch, heads) or (per_row and kc.shape[0] != batch):
        raise ValueError("shape mismatch")
    out = np.full((batch, S), np.nan, dtype=np.float64)
    for t in range(batch):
        L = S if valid_len is None else max(0, min(int(valid_len[t]), S))
        keys = kc[t] if per_row else kc
        dots = q[t] @ keys[:L].T                # [heads, L]: per-head dot products
        relu = np.maximum(dots, 0.0)            # ReLU on each head's product
        out[t, :L] = (w64[t][:, None] * relu).sum(axis=0)   # weight, then sum heads
    return out


def indexer_topk(q_bits, k_bits, w, k, valid_len=None):
    """Top-k positions of each indexer score row.

    Returns (idx [batch, k] int64 in selection order with -1 padding,
    scores [batch, S] float64 as from ``indexer_scores``).
    """
    scores = indexer_scores(q_bits, k_bits, w, valid_len)
    batch, S = scores.shape
    idx = np.full((batch, int(k)), -1, dtype=np.int64)
    for t in range(batch):
        L = S if valid_len is None else max(0, min(int(valid_len[t]), S))
        idx[t] = topk_row(scores[t, :L], k, L)
    return idx, scores
