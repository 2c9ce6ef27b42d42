"""CPU oracle for the sparse-attention selection step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
this package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` (and its ``--impl reference`` arm) may use it.  It shares no
code with the CUDA library under ``sparse_attention_top_ds_b200/csrc``.

Everything here is a plain, slow, single-threaded restatement of what the
selection step computes, in float64:

* ``encoding``   -- IEEE binary32 / bfloat16 bit patterns decoded to float64.
* ``topk``       -- row-wise top-k of given scores: a stable descending sort,
                    ties to the lower index (DeepSelect hub page, the two
                    use-case paragraphs: lightning indexer at topk=512 in
                    bfloat16, sampling over a ~128K vocabulary in float32, and
                    the ``sorted_index`` / ``return_value`` options).
* ``attention``  -- multi-query softmax attention over the selected compressed
                    rows plus a sliding window (NKI pull request, steps table
                    row 4 "Concatenate and attend"), with an optional per-head
                    attention sink.
* ``qproj``      -- the indexer query projection: q = x . Wq^T into 128
                    channels per head, rounded to bfloat16, and the per-head
                    weights w = x . Ww^T (NKI pull request, steps table row 2
                    and the launch list's query-projection GEMV).
* ``indexer``    -- the lightning-indexer score
                    ``score[t,s] = sum_h w[t,h] * max(0, q[t,h,:] . k[s,:])``
                    (NKI pull request "Add DeepSeek-V4 CSA attention kernels",
                    "How the algorithm works", steps table, row 2) followed by
                    the same top-k.

* ``compress``   -- the compressor's 4:1 fold as a gated weighted sum (NKI pull
                    request, steps table row 1).  PARITY UNPINNED: the pages do
                    not give the gate, so the function follows a stated reading.

Every function is pinned by the ``-m "not gpu"`` tests in ``tests/test_oracle_*``
against brute force, closed forms, hand-worked examples under ``tests/golden``
and invariants.  ``compress_fold`` alone is "parity unpinned": its pins check
the stated reading of the gate, which no page fixes.
"""

from .encoding import decode_bf16, decode_f32, NEG_INF_BF16, NEG_INF_F32
from .topk import topk_rows, topk_row
from .indexer import indexer_scores, indexer_topk
from .attention import sparse_attention
from .qproj import qproj, round_bf16
from .compress import compress_fold

__all__ = [
    "decode_bf16", "decode_f32", "NEG_INF_BF16", "NEG_INF_F32",
    "topk_rows", "topk_row", "indexer_scores", "indexer_topk", "sparse_attention", "qproj", "round_bf16", "compress_fold",
]
