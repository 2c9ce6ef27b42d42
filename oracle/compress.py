"""Compressor fold: 4 tokens into 1 by a gated weighted sum (oracle; test
infrastructure only).

PARITY UNPINNED.  The pages name the step but not the gate: NKI pull request
"Add DeepSeek-V4 CSA attention kernels", steps table row 1 ("Compressor"):
the compressor folds 4 tokens into 1 with a gated weighted sum, once every 4
decode steps.  How the gate is computed is not given on any page, so this
function states one reading -- the plainest one that fits "gated weighted
sum" -- and its pins check the function against that reading's closed forms,
not against the pages.

Reading: each of the 4 tokens x_i (rows of width D) gets one gate score
s_i = g . x_i from a gate vector g of width D; the weights are
a = softmax(s_0..s_3); the folded row is sum_i a_i x_i.
"""

import numpy as np

from .encoding import decode_bf16


def compress_fold(rows_bits, gate_bits):
    """float64 folded rows [B, D] from ``rows_bits`` [B, 4, D] and ``gate_bits``
    [D] (bfloat16 patterns)."""
    x = decode_bf16(rows_bits)
    g = decode_bf16(gate_bits)
    B, four, D = x.shape
    if four != 4 or g.shape != (D,):
        raise ValueError("rows must be [B, 4, D] and the gate [D]")
    out = np.zeros((B, D), dtype=np.float64)
    for b in range(B):
        s = x[b] @ g                      # one gate score per token
        a = np.exp(s - s.max())
        a /= a.sum()                      # softmax over the 4 tokens
        out[b] = a @ x[b]                 # the gated weighted sum
    return out
