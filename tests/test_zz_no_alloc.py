"""The allocation-free entry point ds_indexer_topk_noalloc, called through the C ABI.

It exists for callers that cannot call cudaMalloc (an engine that has
reserved all device memory for its own pool, code running under another
framework's allocation-free graph capture, latency-bound paths): its score rows
live in a fixed array inside the library.  Its results must match the regular
ds_indexer_topk, which uses the library's grow-only scratch buffer, within the
tolerance the indexer tests use, on two calls in a row with different inputs
(the fixed array keeps the previous call's contents).  This file runs last so
that a stop-at-first-failure run has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import sparse_attention_top_ds_b200 as ds
from sparse_attention_top_ds_b200 import _native, inputs

pytestmark = pytest.mark.gpu

REL_TOL = 1e-2
NOALLOC_LIMIT = 262144  # batch * S of the fixed array


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _call(fn, qd, kd, wd, vd, k):
    B, H, d = qd.shape
    S = kd.shape[0]
    idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    score = torch.full((B, k), float("nan"), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = fn(ctypes.c_void_p(qd.data_ptr()), ctypes.c_void_p(kd.data_ptr()), ctypes.c_void_p(wd.data_ptr()),
            B, H, d, S, None if vd is None else ctypes.c_void_p(vd.data_ptr()), k,
            ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(score.data_ptr()), stream)
    assert rc == ds.DS_OK, ds.strerror(rc)
    torch.cuda.synchronize()
    assert ds.ds_get_device_status() == ds.DS_OK
    return idx.cpu().numpy(), score.cpu().numpy()


def _compare(a, b):
    (ia, sa), (ib, sb) = a, b
    for t in range(ia.shape[0]):
        m = int((ia[t] >= 0).sum())
        assert int((ib[t] >= 0).sum()) == m
        assert np.all(ia[t, m:] == -1) and np.all(ib[t, m:] == -1)
        assert np.all(np.isneginf(sa[t, m:])) and np.all(np.isneginf(sb[t, m:]))
        if m == 0:
            continue
        assert np.array_equal(np.sort(ia[t, :m]), np.sort(ib[t, :m])), f"row {t}: index sets differ"
        oa, ob = np.argsort(ia[t, :m]), np.argsort(ib[t, :m])
        ra, rb = sa[t, :m][oa].astype(np.float64), sb[t, :m][ob].astype(np.float64)
        assert np.all(np.abs(ra - rb) <= REL_TOL * np.abs(rb) + 1e-6 * max(np.abs(rb).max(), 1e-30))


def test_noalloc_matches_regular_entry_on_two_calls(cuda_device):
    lib = _native.load()
    # call 1: the decode workload (8 rows x 32768 positions, the array's full size)
    q, kc, w, vl = inputs.decode()
    args1 = (_dev_bf16(q), _dev_bf16(kc), torch.from_numpy(w).cuda(), torch.from_numpy(vl).cuda())
    # call 2: another seeded input, fewer positions, a row with no eligible position
    q2, kc2, w2 = inputs.indexer_factors(seed=77, batch=5, n=20000)
    vl2 = np.array([20000, 0, 7, 19999, 12345], dtype=np.int32)
    args2 = (_dev_bf16(q2), _dev_bf16(kc2), torch.from_numpy(w2).cuda(), torch.from_numpy(vl2).cuda())
    for args, k in ((args1, 1024), (args2, 2048)):
        got = _call(lib.ds_indexer_topk_noalloc, *args, k)
        ref = _call(lib.ds_indexer_topk, *args, k)
        _compare(got, ref)


def test_noalloc_rejects_sizes_beyond_the_fixed_array(cuda_device):
    lib = _native.load()
    B, S = 9, NOALLOC_LIMIT // 8      # 9 x 32768 > 262144
    qd = torch.zeros((B, 64, 128), dtype=torch.bfloat16, device="cuda")
    kd = torch.zeros((S, 128), dtype=torch.bfloat16, device="cuda")
    wd = torch.zeros((B, 64), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, 16), dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.ds_indexer_topk_noalloc(ctypes.c_void_p(qd.data_ptr()), ctypes.c_void_p(kd.data_ptr()),
                                     ctypes.c_void_p(wd.data_ptr()), B, 64, 128, S, None, 16,
                                     ctypes.c_void_p(idx.data_ptr()), None, stream)
    assert rc == ds.DS_ERR_ARG
