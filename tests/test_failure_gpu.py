"""Failure detection on the GPU, without a GPU fault.

A planted fault (ds_plant_wait_fault) makes one CTA of the indexer scorer skip
one mbarrier arrival, so that the waits behind it run out after a short limit
(ds_set_wait_limit); the kernel records DS_ERR_TIMEOUT in the status word,
lets its copies land, frees its tensor memory and returns.  The call's outputs
stay well formed (every index -1 or a valid position, every score finite or
-inf), and the next call without the fault returns DS_OK with results that
match the oracle.

The DS_DEBUG build (libdstopk_debug.so) records inputs read on the device
outside their documented range as DS_ERR_RANGE and otherwise behaves as the
release build; it runs in a child process of its own, since one process loads
one build of the library.
"""

import json
import os
import subprocess
import sys
import time

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_top_ds_b200 as ds
from sparse_attention_top_ds_b200 import inputs

from gpu_util import bf16_to_device, f32_to_device, i32_to_device
from test_indexer_gpu import REL_TOL, check_selection

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIMIT_NS = 1_000_000  # 1 ms


def _dev(q, kc, w, vl):
    return bf16_to_device(q), bf16_to_device(kc), f32_to_device(w), i32_to_device(vl)


@pytest.fixture
def short_waits(cuda_device):
    ds.ds_set_wait_limit(LIMIT_NS)
    ds.ds_get_device_status()
    yield
    ds.ds_plant_wait_fault(0)
    ds.ds_set_wait_limit(0)
    ds.ds_get_device_status()


def _check_well_formed(idx, score, vl, S, k):
    for t in range(idx.shape[0]):
        L = max(0, min(int(vl[t]), S))
        sel = idx[t]
        assert np.all((sel == -1) | ((sel >= 0) & (sel < L))), f"row {t}: index out of range"
        got = sel[sel >= 0]
        assert len(np.unique(got)) == len(got), f"row {t}: repeated index"
        assert not np.any(np.isnan(score[t])), f"row {t}: NaN score"


# 8 rows x 32768 keys: every scorer CTA holds several 128-key tiles, so the
# planted skip leaves the MMA warp waiting on its third tile
@pytest.mark.parametrize("entry", ["fused", "noalloc"])
def test_planted_fault_times_out_then_recovers(short_waits, entry):
    B, S, k = 8, 32768, 1024
    q, kc, w, vl = inputs.decode(seed=77, batch=B, S=S, vl_lo=S // 2, vl_hi=S)
    qd, kd, wd, vd = _dev(q, kc, w, vl)
    fn = ds.ds_indexer_topk if entry == "fused" else ds.ds_indexer_topk_noalloc

    ds.ds_plant_wait_fault(1)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    idx, sc = fn(qd, kd, wd, k, valid_len=vd, return_score=True)
    status = ds.ds_get_device_status()
    elapsed = time.perf_counter() - t0
    assert status == ds.DS_ERR_TIMEOUT, ds.strerror(status)
    # the waits gave up after the 1 ms limit, not the default of one second
    assert elapsed < 0.5, f"planted call took {elapsed:.3f} s"
    _check_well_formed(idx.cpu().numpy(), sc.cpu().numpy(), vl, S, k)

    # the next call (no fault planted) is clean and correct
    idx, sc = fn(qd, kd, wd, k, valid_len=vd, return_score=True)
    assert ds.ds_get_device_status() == ds.DS_OK
    check_selection(q, kc, w, vl, k, idx.cpu().numpy(), sc.cpu().numpy())


def test_planted_fault_in_the_scorer_leaves_minus_inf(short_waits):
    # the score rows of a timed-out launch: the positions the faulty CTA did
    # not reach hold -inf, every other position its score
    B, H, S = 8, 64, 32768
    q, kc, w = inputs.indexer_factors(seed=78, batch=B, n=S, heads=H)
    qd, kd, wd = bf16_to_device(q), bf16_to_device(kc), f32_to_device(w)
    ref = oracle.indexer_scores(q, kc, w)
    ds.ds_plant_wait_fault(1)
    out = ds.ds_indexer_score(qd, kd, wd)
    assert ds.ds_get_device_status() == ds.DS_ERR_TIMEOUT
    got = out.cpu().numpy().astype(np.float64)
    lost = np.isneginf(got)
    assert lost.any(), "the planted fault left every score in place"
    assert lost.sum() < got.size // 4, "far more positions lost than one CTA holds"
    ok = ~lost
    tol = REL_TOL * np.abs(ref) + 1e-6 * np.maximum(np.abs(ref).max(axis=1, keepdims=True), 1e-30)
    assert np.all(np.abs(got[ok] - ref[ok]) <= tol[ok])
    out = ds.ds_indexer_score(qd, kd, wd)
    assert ds.ds_get_device_status() == ds.DS_OK
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= tol)


def test_fault_is_armed_per_launch(short_waits):
    # two planted launches, then none: the third call is clean
    B, S, k = 8, 32768, 512
    q, kc, w, vl = inputs.decode(seed=79, batch=B, S=S, vl_lo=S // 2, vl_hi=S)
    qd, kd, wd, vd = _dev(q, kc, w, vl)
    ds.ds_plant_wait_fault(2)
    for _ in range(2):
        ds.ds_indexer_topk(qd, kd, wd, k, valid_len=vd)
        assert ds.ds_get_device_status() == ds.DS_ERR_TIMEOUT
    idx, _ = ds.ds_indexer_topk(qd, kd, wd, k, valid_len=vd)
    assert ds.ds_get_device_status() == ds.DS_OK
    check_selection(q, kc, w, vl, k, idx.cpu().numpy(), None)


_CHILD = r"""
import json, sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import sparse_attention_top_ds_b200 as ds
from sparse_attention_top_ds_b200 import inputs
from gpu_util import bf16_to_device, f32_to_device, i32_to_device
torch.cuda.set_device(0)
res = {"debug": ds.ds_debug_build()}
B, S, k = 6, 5000, 300
q, kc, w = inputs.indexer_factors(seed=81, batch=B, n=S, heads=64)
qd, kd, wd = bf16_to_device(q), bf16_to_device(kc), f32_to_device(w)
vl_bad = np.array([S + 5, -3, 4000, S, 0, 2500], dtype=np.int32)
vl_ok = np.clip(vl_bad, 0, S).astype(np.int32)
a, _ = ds.ds_indexer_topk(qd, kd, wd, k, valid_len=i32_to_device(vl_bad))
res["indexer_bad"] = ds.ds_get_device_status()
b, _ = ds.ds_indexer_topk(qd, kd, wd, k, valid_len=i32_to_device(vl_ok))
res["indexer_ok"] = ds.ds_get_device_status()
res["same_as_clamped"] = bool(np.array_equal(np.sort(a.cpu().numpy(), 1), np.sort(b.cpu().numpy(), 1)))
x = torch.randn(4, 8192, device="cuda")
ds.ds_topk(x, 64, valid_len=i32_to_device(np.array([8192, 9000, 10, 0], dtype=np.int32)))
res["topk_bad"] = ds.ds_get_device_status()
ds.ds_topk(x, 64, valid_len=i32_to_device(np.array([8192, 8192, 10, 0], dtype=np.int32)))
res["topk_ok"] = ds.ds_get_device_status()
print("RESULT " + json.dumps(res))
"""


def _run_child(lib):
    env = dict(os.environ)
    env["DS_TOPK_LIB"] = lib
    out = subprocess.run([sys.executable, "-c", _CHILD, ROOT], env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-4000:]
    line = [ln for ln in out.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    return json.loads(line[len("RESULT "):])


def test_debug_build_flags_out_of_range_inputs(cuda_device):
    from sparse_attention_top_ds_b200 import build
    r = _run_child(build.LIB_DEBUG)
    assert r["debug"] is True
    assert r["indexer_bad"] == ds.DS_ERR_RANGE and r["indexer_ok"] == ds.DS_OK
    assert r["topk_bad"] == ds.DS_ERR_RANGE and r["topk_ok"] == ds.DS_OK
    assert r["same_as_clamped"], "the debug build must clamp exactly as the release build"


def test_release_build_clamps_without_a_word(cuda_device):
    from sparse_attention_top_ds_b200 import build
    r = _run_child(build.LIB)
    assert r["debug"] is False
    assert r["indexer_bad"] == ds.DS_OK and r["topk_bad"] == ds.DS_OK
    assert r["same_as_clamped"]
