"""Row-wise top-k of given scores (oracle; test infrastructure only).

What is computed (DeepSelect hub page, use-case paragraphs: select the most
relevant positions of each row, topk=512 in bfloat16 for the lightning indexer,
float32 over a ~129K vocabulary for sampling; options ``sorted_index`` and
``return_value``):

for each row t, with L = min(valid_len[t], n):
  1. decode the first L stored values exactly to float64;
  2. order the positions 0..L-1 by value, largest first, with equal values kept
     in ascending position order (a stable descending sort);
  3. the first m = min(k, L) positions are the selection;
  4. the returned value of a selected position is its stored bit pattern,
     copied unchanged;
  5. slots m..k-1 are padding: index -1, value -inf.

Readings where the pages are silent:
  * ties go to the lower index;
  * -0.0 and +0.0 are equal (the index decides);
  * every NaN ranks above +inf and all NaNs are equal (the index decides);
  * valid_len is a prefix length; None means n;
  * without ``sorted_index`` the order of the selection is unspecified and is
    compared as a set; with it, indices come in ascending order.
"""

import numpy as np

from .encoding import decode_bf16, decode_f32, NEG_INF_BF16, NEG_INF_F32


def topk_row(values, k, valid_len=None):
    """Selection order for one row of float64 values.

    Returns an int64 array of length k: the selected positions in descending
    value order (ties by ascending position), then -1 padding.
    """
    values = np.asarray(values, dtype=np.float64)
    n = values.shape[0]
    L = n if valid_len is None else max(0, min(int(valid_len), n))
    v = values[:L]
    nan = np.isnan(v)
    # Sort keys, most significant last (numpy.lexsort convention):
    #   class 0 = NaN (ranks above everything), class 1 = numbers;
    #   within numbers, the negated value ascending (= value descending),
    #   with -0.0 folded onto +0.0 so the two zeros compare equal;
    #   finally the position, ascending, so ties keep index order.
    neg = np.where(nan | (v == 0.0), 0.0, -v)
    cls = np.where(nan, 0, 1)
    order = np.lexsort((np.arange(L), neg, cls))
    m = min(int(k), L)
    out = np.full(int(k), -1, dtype=np.int64)
    out[:m] = order[:m]
    return out


def topk_rows(bits, dtype, k, valid_len=None, sorted_index=False):
    """Top-k of every row of a [batch, n] array of stored scores.

    ``bits``      uint16 bfloat16 patterns when dtype == "bf16";
                  float32 values or uint32 patterns when dtype == "f32".
    ``valid_len`` None, or one prefix length per row.
    Returns (idx [batch, k] int64, val [batch, k] stored bit patterns as
    uint16 / uint32).  Without ``sorted_index`` each row is in selection order
    (value descending, ties by ascending index); with it, the selected indices
    are in ascending order.  Padding slots hold index -1 and the -inf pattern.
    """
    if dtype == "bf16":
        raw = np.asarray(bits).astype(np.uint16)
        dec = decode_bf16(raw)
        pad_val, vdt = NEG_INF_BF16, np.uint16
    elif dtype == "f32":
        a = np.asarray(bits)
        raw = a.view(np.uint32) if a.dtype == np.float32 else a.astype(np.uint32)
        dec = decode_f32(raw)
        pad_val, vdt = NEG_INF_F32, np.uint32
    else:
        raise ValueError("dtype must be 'bf16' or 'f32'")
    if raw.ndim != 2:
        raise ValueError("scores must be [batch, n]")
    batch, n = raw.shape
    idx = np.full((batch, int(k)), -1, dtype=np.int64)
    val = np.full((batch, int(k)), pad_val, dtype=vdt)
    for t in range(batch):
        vl = None if valid_len is None else int(valid_len[t])
        sel = topk_row(dec[t], k, vl)
        m = int((sel >= 0).sum())
        chosen = sel[:m]
        if sorted_index:
            chosen = np.sort(chosen)
        idx[t, :m] = chosen
        val[t, :m] = raw[t, chosen]
    return idx, val
