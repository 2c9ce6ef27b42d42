"""B200-native selection step of DeepSeek-style sparse attention.

The work happens in libdstopk.so (CUDA kernels for sm_100a behind the C ABI in
include/ds_topk.h); this package is its Python binding plus seeded input
generators:

    ds_topk            top-k of bfloat16 / float32 score rows
    ds_indexer_score   lightning-indexer score rows (tcgen05 tensor cores)
    ds_indexer_topk    indexer score + top-k: the scorer also counts every row's key
                       histogram, from which the selection takes its threshold
    ds_indexer_topk_noalloc  the same without any device allocation (two launches,
                       score rows in a fixed array of the library)
    ds_indexer_qproj   the indexer query projection (queries and per-head weights)
    ds_sparse_attention  multi-query attention over the selected rows plus a
                       sliding window (tcgen05 tensor cores)
"""

from ._native import (  # noqa: F401
    DS_F32, DS_BF16, DS_OK, DS_ERR_ARG, DS_ERR_CUDA, DS_ERR_TIMEOUT, DS_ERR_UNSUPPORTED,
    DS_ERR_NOMEM, DS_ERR_RANGE, DS_MAX_K, DS_INDEXER_DIM, DS_INDEXER_MAX_HEADS, DS_ATTN_MAX_DIM, DS_ATTN_MAX_WINDOW,
    DS_ATTN_MAX_HEADS, DsError,
    ds_topk, ds_indexer_score, ds_indexer_topk, ds_indexer_topk_noalloc, ds_indexer_topk_ex, ds_indexer_qproj, ds_compress_fold, ds_sparse_attention, ds_get_device_status,
    ds_release, ds_set_wait_limit, ds_plant_wait_fault, ds_debug_build, ds_debug_stash_stamps, ds_read_floor,
    strerror, load, lib_path, DEBUG_LIB_PATH,
)
