"""GPU parity of ds_sparse_attention with the float64 oracle.

The bar, from the arithmetic (the softmax weights are rounded to bfloat16
twice, at most 2^-8 relative each, and the output once more): per batch row,
max |out - out_ref| <= 1e-2 * max |value of an attended row|, and
|lse - lse_ref| <= 5e-3; -inf lse and zero output exactly where nothing is
attended.  Inputs come from sparse_attention_top_ds_b200.inputs, expected
values from oracle.sparse_attention.
"""

import math

import numpy as np
import pytest
import torch

import sparse_attention_top_ds_b200 as ds
from oracle import sparse_attention as oracle_attention
from sparse_attention_top_ds_b200 import inputs

from gpu_util import bf16_to_device, f32_to_device, i32_to_device, bits_of

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2   # times the largest |value| among the attended rows of the batch row
LSE_TOL = 5e-3


def _dec(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _to_device(a, dev):
    t = dict(q=bf16_to_device(a["q"], dev), kv=bf16_to_device(a["kv"], dev),
             idx=i32_to_device(a["idx"], dev) if a["idx"].shape[1] > 0 else None,
             win=bf16_to_device(a["win"], dev) if a["win"].shape[1] > 0 else None,
             win_len=i32_to_device(a["win_len"], dev),
             sink=f32_to_device(a["sink"], dev) if a["sink"] is not None else None)
    return t


def _run(a, dev, scale, use_win_len=True):
    t = _to_device(a, dev)
    out, lse = ds.ds_sparse_attention(t["q"], t["kv"], t["idx"], scale=scale, win=t["win"],
                                      win_len=t["win_len"] if use_win_len else None, sink=t["sink"],
                                      return_lse=True)
    torch.cuda.synchronize()
    return _dec(bits_of(out)), lse.cpu().numpy().astype(np.float64)


def _check(a, out, lse, scale, rows=None):
    W = a["win"].shape[1]
    ref_out, ref_lse = oracle_attention(a["q"], a["kv"], a["idx"], scale, win=a["win"] if W else None,
                                        win_len=a["win_len"], sink=a["sink"])
    kv = _dec(a["kv"])
    win = _dec(a["win"])
    B = a["q"].shape[0]
    for b in (range(B) if rows is None else rows):
        cache = kv if kv.ndim == 2 else kv[b]
        sel = [int(i) for i in a["idx"][b] if 0 <= int(i) < cache.shape[0]]
        wl = max(0, min(int(a["win_len"][b]), W))
        vals = [np.abs(cache[sel]).max()] if sel else []
        if wl:
            vals.append(np.abs(win[b, :wl]).max())
        if not vals:
            assert np.all(out[b] == 0.0), f"row {b}: nothing attended but output not zero"
            if a["sink"] is None:
                assert np.all(np.isneginf(lse[b])), f"row {b}: lse"
            else:
                assert np.allclose(lse[b], a["sink"].astype(np.float64), atol=1e-6, rtol=0)
            continue
        vmax = max(vals)
        err = np.abs(out[b] - ref_out[b]).max()
        assert err <= OUT_TOL * vmax, f"row {b}: max |out - ref| = {err:.3e} > {OUT_TOL} * {vmax:.3f}"
        lerr = np.abs(lse[b] - ref_lse[b]).max()
        assert lerr <= LSE_TOL, f"row {b}: max |lse - ref| = {lerr:.3e}"


SMALL = [
    # B, H, d, T, k, W, shared, sink, holes, win_len
    (3, 128, 512, 3000, 300, 128, True, True, 0.2, [128, 5, 0]),
    (2, 40, 128, 500, 77, 0, True, False, 0.0, None),
    (2, 160, 256, 900, 64, 64, False, True, 0.1, [64, 33]),
    (1, 128, 64, 100, 1, 0, True, True, 0.0, None),
    (2, 64, 192, 700, 130, 17, False, False, 0.3, [17, 2]),
    (2, 128, 320, 800, 200, 40, True, True, 0.0, [40, 40]),
    (1, 128, 512, 5000, 0, 128, True, True, 0.0, [100]),
    (4, 8, 512, 2048, 2048, 0, False, True, 0.05, None),
]


@pytest.mark.parametrize("case", SMALL, ids=[f"B{c[0]}H{c[1]}d{c[2]}k{c[4]}W{c[5]}" for c in SMALL])
def test_matches_oracle(case, cuda_device):
    B, H, d, T, k, W, shared, sink, holes, wl = case
    a = inputs.attention(seed=100 + H + d + k, batch=B, heads=H, d=d, T=T, k=k, W=W, shared_cache=shared,
                         vl_lo=min(T, 50), vl_hi=T, sink=sink, holes=holes, win_len=wl)
    scale = 1.0 / math.sqrt(d)
    out, lse = _run(a, cuda_device, scale)
    _check(a, out, lse, scale)


def test_repeated_slots(cuda_device):
    # a row picked by several slots is attended once per slot; the repeats sit in
    # other 64-row chunks than the first pick, and one row repeats 40 times
    a = inputs.attention(seed=8, batch=2, heads=128, d=512, T=3000, k=400, W=64, shared_cache=False,
                         vl_lo=1000, vl_hi=3000, holes=0.0)
    idx = a["idx"]
    idx[0, 300:340] = idx[0, 5]
    idx[1, 100:400:3] = idx[1, 100:200]
    scale = 2.0 / math.sqrt(512)
    out, lse = _run(a, cuda_device, scale)
    _check(a, out, lse, scale)


def test_sharp_softmax(cuda_device):
    # a large score factor: the chunk maxima differ by many units, exercising
    # the rescaling of the combine step
    a = inputs.attention(seed=7, batch=2, heads=128, d=512, T=4000, k=500, W=128, shared_cache=True,
                         vl_lo=1000, vl_hi=4000, holes=0.1)
    scale = 6.0 / math.sqrt(512)
    out, lse = _run(a, cuda_device, scale)
    _check(a, out, lse, scale)


def test_nothing_attended(cuda_device):
    a = inputs.attention(seed=8, batch=3, heads=128, d=256, T=100, k=70, W=16, shared_cache=True,
                         vl_lo=100, vl_hi=100, win_len=[0, 0, 3])
    a["idx"][:2] = -1
    a["idx"][0, 5] = 100          # past the cache: skipped as well
    scale = 1 / 16
    out, lse = _run(a, cuda_device, scale)
    _check(a, out, lse, scale)
    a["sink"] = None
    out, lse = _run(a, cuda_device, scale)
    _check(a, out, lse, scale)
    assert np.all(np.isneginf(lse[:2]))


def test_without_win_len_the_whole_window_counts(cuda_device):
    a = inputs.attention(seed=9, batch=2, heads=128, d=128, T=1000, k=100, W=50, shared_cache=True,
                         vl_lo=500, vl_hi=1000)
    out, lse = _run(a, cuda_device, 0.1, use_win_len=False)
    a["win_len"] = np.full(2, 50, dtype=np.int32)
    _check(a, out, lse, 0.1)


def test_decode_workload_full_size(cuda_device):
    """8 tokens x 128 heads x d = 512, 32768-row cache per batch row, k = 1024
    selected rows plus a window of 128 and a sink: every output checked."""
    a = inputs.attention()
    scale = 1.0 / math.sqrt(512)
    out, lse = _run(a, cuda_device, scale)
    _check(a, out, lse, scale)


def test_many_rows_run_in_pieces(cuda_device):
    # 1024 rows x 34 chunks of weight and row tiles (about 2.8 MiB a row)
    # exceed the 512 MiB scratch cap, so the call runs in several pieces of
    # about 180 rows; rows from several pieces are checked
    a = inputs.attention(seed=10, batch=1024, heads=128, d=512, T=8192, k=2048, W=128, shared_cache=True,
                         vl_lo=4096, vl_hi=8192)
    scale = 1.0 / math.sqrt(512)
    out, lse = _run(a, cuda_device, scale)
    rows = [0, 1, 181, 182, 500, 906, 907, 1023]
    sub = dict(a)
    sub["q"], sub["idx"], sub["win"], sub["win_len"] = a["q"][rows], a["idx"][rows], a["win"][rows], a["win_len"][rows]
    _check(sub, out[rows], lse[rows], scale)


def test_chained_after_the_selection_on_one_stream(cuda_device):
    """Slots written by ds_indexer_topk and read by the attention kernel right
    after it (programmatic dependent launch): the result equals the one from
    the same slots read after a synchronisation."""
    q, kc, w, vl = inputs.decode(seed=11, batch=4, S=8192, vl_lo=2000, vl_hi=8192)
    a = inputs.attention(seed=12, batch=4, heads=128, d=512, T=8192, k=1024, W=128, shared_cache=True)
    t = _to_device(a, cuda_device)
    iq, ik = bf16_to_device(q, cuda_device), bf16_to_device(kc, cuda_device)
    iw, ivl = f32_to_device(w, cuda_device), i32_to_device(vl, cuda_device)
    idx = torch.empty((4, 1024), dtype=torch.int32, device=cuda_device)
    s = torch.cuda.Stream(cuda_device)
    with torch.cuda.stream(s):
        for _ in range(3):
            idx.fill_(-1)
            ds.ds_indexer_topk(iq, ik, iw, 1024, valid_len=ivl, out_idx=idx)
            chained = ds.ds_sparse_attention(t["q"], t["kv"], idx, win=t["win"], win_len=t["win_len"],
                                             sink=t["sink"])
    s.synchronize()
    direct = ds.ds_sparse_attention(t["q"], t["kv"], idx.clone(), win=t["win"], win_len=t["win_len"],
                                    sink=t["sink"])
    torch.cuda.synchronize()
    assert torch.equal(chained.view(torch.int16), direct.view(torch.int16))


def test_graph_replay(cuda_device):
    a = inputs.attention(seed=13, batch=8, heads=128, d=512, T=4096, k=1024, W=128, shared_cache=True,
                         vl_lo=2048, vl_hi=4096)
    t = _to_device(a, cuda_device)
    out = torch.empty((8, 128, 512), dtype=torch.bfloat16, device=cuda_device)
    ds.ds_sparse_attention(t["q"], t["kv"], t["idx"], win=t["win"], win_len=t["win_len"], sink=t["sink"], out=out)
    torch.cuda.synchronize()
    first = out.clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(cuda_device)
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            ds.ds_sparse_attention(t["q"], t["kv"], t["idx"], win=t["win"], win_len=t["win_len"],
                                   sink=t["sink"], out=out)
    out.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), first.view(torch.int16))
    assert ds.ds_get_device_status() == ds.DS_OK


def test_largest_slots_and_window(cuda_device):
    """k = 2048 slots plus the largest window (4096 rows): 96 chunks of 64 rows
    per batch row, so the weighted-sum kernel runs its 2-chunk stages with the
    largest statistics block; d = 512, 160 heads (two head tiles)."""
    a = inputs.attention(seed=14, batch=2, heads=160, d=512, T=6000, k=2048, W=4096, shared_cache=False,
                         vl_lo=3000, vl_hi=6000, holes=0.02, win_len=[4096, 1234])
    scale = 1.0 / math.sqrt(512)
    out, lse = _run(a, cuda_device, scale)
    _check(a, out, lse, scale)
