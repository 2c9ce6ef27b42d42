"""The allocation-free entry point ds_indexer_topk_noalloc, called through the C ABI.

It exists for callers that cannot call cudaMalloc (an engine that has
reserved all device memory for its own pool, code running under another
framework's allocation-free graph capture, latency-bound paths): its score rows
live in a fixed array inside the library.  Its results must match the regular
ds_indexer_topk, which uses the library's grow-only scratch buffer, within the
tolerance the indexer tests use, on two calls in a row with different inputs
(the fixed array keeps the previous call's contents), and the oracle's
selection.  Two child processes show that the first call allocates nothing:
with every module loaded up front and the library's device set-up done, the
device's free memory is the same before and after it (while a first regular
call takes its scratch); and a first call captured into a CUDA graph -- where
a cudaMalloc would end the capture with an error -- replays correctly, at
batch * S past anything the regular scratch holds at that point.  This file
runs last so that a stop-at-first-failure run has already run every other
test.
"""

import ctypes
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import sparse_attention_top_ds_b200 as ds
from sparse_attention_top_ds_b200 import _native, inputs

from test_indexer_gpu import check_selection

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


def test_noalloc_matches_the_oracle(cuda_device):
    lib = _native.load()
    for seed, B, S, k, vl in ((91, 8, 32768, 1024, None), (92, 6, 9000, 2048, [9000, 0, 1, 8999, 4500, -2]),
                              (93, 64, 4096, 512, None)):
        q, kc, w = inputs.indexer_factors(seed=seed, batch=B, n=S)
        vln = None if vl is None else np.array(vl, dtype=np.int32)
        args = (_dev_bf16(q), _dev_bf16(kc), torch.from_numpy(w).cuda(),
                None if vln is None else torch.from_numpy(vln).cuda())
        idx, score = _call(lib.ds_indexer_topk_noalloc, *args, k)
        check_selection(q, kc, w, vln, k, idx, score)


_CHILD_MEMINFO = r"""
import json, sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1])
import sparse_attention_top_ds_b200 as ds
from sparse_attention_top_ds_b200 import inputs
torch.cuda.set_device(0)
q, kc, w, vl = inputs.decode()
bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
qd, kd, wd, vd = bf(q), bf(kc), torch.from_numpy(w).cuda(), torch.from_numpy(vl).cuda()
idx = torch.empty((8, 1024), dtype=torch.int32, device="cuda")
sc = torch.empty((8, 1024), dtype=torch.float32, device="cuda")
# the library's one-time device set-up (kernel attributes, the status word's
# address); the CUDA driver reserves a few MiB of its own on that first use
ds.ds_get_device_status()
torch.cuda.synchronize()
free0 = torch.cuda.mem_get_info()[0]
ds.ds_indexer_topk_noalloc(qd, kd, wd, 1024, valid_len=vd, return_score=True, out_idx=idx, out_score=sc)
torch.cuda.synchronize()
free1 = torch.cuda.mem_get_info()[0]
status = ds.ds_get_device_status()
ds.ds_indexer_topk(qd, kd, wd, 1024, valid_len=vd, out_idx=idx)
torch.cuda.synchronize()
free2 = torch.cuda.mem_get_info()[0]
print("RESULT " + json.dumps({"free0": free0, "free1": free1, "free2": free2, "status": status}))
"""

_CHILD_CAPTURE = r"""
import json, sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import sparse_attention_top_ds_b200 as ds
from sparse_attention_top_ds_b200 import inputs
from test_indexer_gpu import check_selection
torch.cuda.set_device(0)
bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
# a small regular call first: the library's own scratch now holds 2 x 1000 scores
qs, ks, ws = inputs.indexer_factors(seed=3, batch=2, n=1000)
ds.ds_indexer_topk(bf(qs), bf(ks), torch.from_numpy(ws).cuda(), 10)
torch.cuda.synchronize()
# then the first allocation-free call, 8 x 32768 positions, inside a graph capture
q, kc, w, vl = inputs.decode(seed=5)
qd, kd, wd, vd = bf(q), bf(kc), torch.from_numpy(w).cuda(), torch.from_numpy(vl).cuda()
idx = torch.full((8, 1024), -7, dtype=torch.int32, device="cuda")
sc = torch.empty((8, 1024), dtype=torch.float32, device="cuda")
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g, capture_error_mode="thread_local"):
    ds.ds_indexer_topk_noalloc(qd, kd, wd, 1024, valid_len=vd, return_score=True, out_idx=idx, out_score=sc,
                               stream=torch.cuda.current_stream())
g.replay()
torch.cuda.synchronize()
status = ds.ds_get_device_status()
check_selection(q, kc, w, vl, 1024, idx.cpu().numpy(), sc.cpu().numpy())
print("RESULT " + json.dumps({"status": status}))
"""


def _child(code, extra_env=None):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ)
    env.update(extra_env or {})
    out = subprocess.run([sys.executable, "-c", code, root], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-4000:]
    line = [ln for ln in out.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    return json.loads(line[len("RESULT "):])


def test_first_noalloc_call_leaves_free_memory_unchanged(cuda_device):
    r = _child(_CHILD_MEMINFO, {"CUDA_MODULE_LOADING": "EAGER"})
    assert r["status"] == ds.DS_OK
    assert r["free1"] == r["free0"], f"the first allocation-free call took {r['free0'] - r['free1']} bytes"
    # the control: the regular entry point's first call does allocate its scratch
    assert r["free2"] < r["free1"]


def test_first_noalloc_call_captures_into_a_graph(cuda_device):
    r = _child(_CHILD_CAPTURE)
    assert r["status"] == ds.DS_OK
