"""GPU parity of ds_indexer_score and ds_indexer_topk (through the C ABI) with
the float64 oracle.

Bars (products are bf16 x bf16 accumulated in float32):
  * scores: |gpu - oracle| <= 1e-2 * |oracle| + 1e-6 * rowmax, and the tighter
    float32 accumulation bound (d + H) * 2^-23 * sum|w * relu(q.k)| ... checked
    as 1e-4 relative on the row scale;
  * exact-arithmetic inputs (small integer q, k; power-of-two w): every float32
    partial sum is exact, so scores match bit for bit and the selected index
    sets match exactly;
  * selection on random inputs: min(k, valid_len) distinct in-range indices,
    each with oracle score >= the oracle's k-th value - 1e-2 * |k-th value|, and
    returned scores within 1e-2 relative of the oracle's.
"""

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_top_ds_b200 as ds
from sparse_attention_top_ds_b200 import inputs
from gpu_util import bf16_to_device, f32_to_device, i32_to_device

pytestmark = pytest.mark.gpu

REL_TOL = 1e-2


def dev_inputs(q, kc, w, vl):
    return (bf16_to_device(q), bf16_to_device(kc), f32_to_device(w),
            None if vl is None else i32_to_device(vl))


def check_scores(q, kc, w, vl, strict=True):
    qd, kd, wd, vd = dev_inputs(q, kc, w, vl)
    got = ds.ds_indexer_score(qd, kd, wd, valid_len=vd).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    assert ds.ds_get_device_status() == ds.DS_OK
    ref = oracle.indexer_scores(q, kc, w, vl)
    B, S = ref.shape
    for t in range(B):
        L = S if vl is None else max(0, min(int(vl[t]), S))
        assert np.all(np.isneginf(got[t, L:])), f"row {t}: positions past valid_len must be -inf"
        if L == 0:
            continue
        r, g = ref[t, :L], got[t, :L]
        scale = max(np.abs(r).max(), 1e-30)
        err = np.abs(g - r)
        assert np.all(err <= REL_TOL * np.abs(r) + 1e-6 * scale), f"row {t}: max err {err.max()}"
        if strict:
            assert err.max() <= 1e-4 * scale, f"row {t}: error {err.max() / scale} of the row scale"
    return got, ref


def check_selection(q, kc, w, vl, k, idx, score):
    ref = oracle.indexer_scores(q, kc, w, vl)
    B, S = ref.shape
    for t in range(B):
        L = S if vl is None else max(0, min(int(vl[t]), S))
        m = min(k, L)
        sel = idx[t]
        assert int((sel >= 0).sum()) == m and np.all(sel[m:] == -1), f"row {t}: count / padding"
        s = sel[:m]
        assert len(np.unique(s)) == m and np.all((s >= 0) & (s < L)), f"row {t}: distinct in-range"
        if m == 0:
            continue
        vk = np.sort(ref[t, :L])[::-1][m - 1]
        assert np.all(ref[t, s] >= vk - REL_TOL * abs(vk)), f"row {t}: a selected score is below the k-th"
        if score is not None:
            rs = ref[t, s]
            assert np.all(np.abs(score[t, :m] - rs) <= REL_TOL * np.abs(rs) + 1e-6 * max(abs(vk), 1e-30))
            assert np.all(np.isneginf(score[t, m:]))


# ---------------------------------------------------------------- scores

@pytest.mark.parametrize("B,H,S", [(1, 64, 128), (3, 64, 1000), (8, 64, 4096), (9, 64, 777),
                                   (5, 32, 300), (2, 16, 256), (4, 8, 129), (3, 1, 200), (2, 48, 260)])
def test_scores_random(cuda_device, B, H, S):
    q, kc, w = inputs.indexer_factors(seed=100 + B * H + S, batch=B, n=S, heads=H)
    check_scores(q, kc, w, None)


def test_scores_valid_len(cuda_device):
    q, kc, w = inputs.indexer_factors(seed=5, batch=8, n=3000, heads=64)
    vl = np.array([0, 1, 127, 128, 129, 2999, 3000, 5000], dtype=np.int32)
    check_scores(q, kc, w, vl)


def exact_inputs(seed, B, H, S):
    g = np.random.default_rng(seed)
    q = inputs.f32_to_bf16_bits(g.integers(-4, 5, size=(B, H, 128)).astype(np.float32))
    kc = inputs.f32_to_bf16_bits(g.integers(-4, 5, size=(S, 128)).astype(np.float32))
    w = g.choice(np.array([0.25, 0.5, 1.0, 2.0], dtype=np.float32), size=(B, H))
    return q, kc, w


@pytest.mark.parametrize("B,H,S", [(8, 64, 2048), (13, 64, 700), (2, 64, 33), (8, 32, 500)])
def test_scores_exact_arithmetic(cuda_device, B, H, S):
    q, kc, w = exact_inputs(B * 7 + S, B, H, S)
    got, ref = check_scores(q, kc, w, None)
    assert np.array_equal(got, ref), "exact-arithmetic scores must match bit for bit"


# ---------------------------------------------------------------- selection

@pytest.mark.parametrize("B,H,S,k", [(8, 64, 2048, 1024), (13, 64, 700, 100), (8, 32, 500, 499)])
def test_topk_exact_arithmetic(cuda_device, B, H, S, k):
    q, kc, w = exact_inputs(B * 11 + S, B, H, S)
    qd, kd, wd, _ = dev_inputs(q, kc, w, None)
    idx, score = ds.ds_indexer_topk(qd, kd, wd, k, return_score=True)
    ref_idx, ref_scores = oracle.indexer_topk(q, kc, w, k)
    idx = idx.cpu().numpy()
    score = score.cpu().numpy()
    for t in range(B):
        m = int((ref_idx[t] >= 0).sum())
        assert np.array_equal(np.sort(idx[t, :m]), np.sort(ref_idx[t, :m])), f"row {t}"
        assert np.array_equal(score[t, :m].astype(np.float64), ref_scores[t, idx[t, :m]])


def test_decode_8x64x128_vs_32768_k1024(cuda_device):
    q, kc, w, vl = inputs.decode()
    qd, kd, wd, vd = dev_inputs(q, kc, w, vl)
    idx, score = ds.ds_indexer_topk(qd, kd, wd, 1024, valid_len=vd, return_score=True)
    torch.cuda.synchronize()
    assert ds.ds_get_device_status() == ds.DS_OK
    check_selection(q, kc, w, vl, 1024, idx.cpu().numpy(), score.cpu().numpy())


def test_prefill_4096_rows_sampled(cuda_device):
    q, kc, w, vl = inputs.prefill()
    qd, kd, wd, vd = dev_inputs(q, kc, w, vl)
    idx, score = ds.ds_indexer_topk(qd, kd, wd, 2048, valid_len=vd, return_score=True)
    torch.cuda.synchronize()
    assert ds.ds_get_device_status() == ds.DS_OK
    rows = inputs.sample_rows(inputs.SEED_PREFILL, q.shape[0], 64)
    check_selection(q[rows], kc, w[rows], vl[rows], 2048, idx.cpu().numpy()[rows], score.cpu().numpy()[rows])
    # every row: min(k, valid_len) distinct in-range indices
    allidx = idx.cpu().numpy()
    assert np.all((allidx >= 0) & (allidx < vl[:, None]))
    srt = np.sort(allidx, axis=1)
    assert np.all(np.diff(srt, axis=1) > 0)


@pytest.mark.parametrize("B,H,S,k", [(3, 64, 1000, 2048), (9, 64, 5000, 64), (1, 64, 300, 1), (6, 16, 4000, 512)])
def test_topk_valid_len_and_padding(cuda_device, B, H, S, k):
    q, kc, w = inputs.indexer_factors(seed=B + S + k, batch=B, n=S, heads=H)
    g = np.random.default_rng(B)
    vl = g.integers(-2, S + 10, size=B).astype(np.int32)
    vl[0] = 0
    qd, kd, wd, vd = dev_inputs(q, kc, w, vl)
    idx, score = ds.ds_indexer_topk(qd, kd, wd, k, valid_len=vd, return_score=True)
    check_selection(q, kc, w, vl, k, idx.cpu().numpy(), score.cpu().numpy())


def test_indexer_argument_errors(cuda_device):
    q = torch.zeros((2, 64, 64), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((100, 64), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((2, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(ds.DsError):
        ds.ds_indexer_score(q, kc, w)            # d != 128
    q = torch.zeros((2, 65, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((100, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((2, 65), dtype=torch.float32, device="cuda")
    with pytest.raises(ds.DsError):
        ds.ds_indexer_topk(q, kc, w, 10)         # heads > 64


# ---------------------------------------------------------------- the fused path: whole rows and split rows
#
# ds_indexer_topk scores and selects in one launch.  A CTA group that owns its
# rows whole (many rows, as in prefill) selects them itself; rows split over
# several CTAs (few rows, as in decode) are selected by the group's last CTA from
# the histograms every CTA added up.  ds_indexer_topk_noalloc runs the same
# scorer arithmetic as two launches (scores to a buffer, then ds_topk), so both
# must select the same positions and return the same scores.


def _same_selection(a_idx, a_sc, b_idx, b_sc):
    for t in range(a_idx.shape[0]):
        assert np.array_equal(np.sort(a_idx[t]), np.sort(b_idx[t])), f"row {t}"
        oa, ob = np.argsort(a_idx[t]), np.argsort(b_idx[t])
        assert np.array_equal(a_sc[t][oa], b_sc[t][ob]), f"row {t}: scores"


@pytest.mark.parametrize("B,S,k", [(8, 32768, 1024), (2, 20000, 2048), (1, 5000, 64), (5, 9000, 700)])
def test_fused_matches_two_launch_path(cuda_device, B, S, k):
    q, kc, w, vl = inputs.decode(seed=31 + B, batch=B, S=S, vl_lo=min(4096, S // 2), vl_hi=S)
    qd, kd, wd, vd = dev_inputs(q, kc, w, vl)
    fused, fs = ds.ds_indexer_topk(qd, kd, wd, k, valid_len=vd, return_score=True)
    torch.cuda.synchronize()
    two, ts = ds.ds_indexer_topk_noalloc(qd, kd, wd, k, valid_len=vd, return_score=True)
    torch.cuda.synchronize()
    assert ds.ds_get_device_status() == ds.DS_OK
    _same_selection(fused.cpu().numpy(), fs.cpu().numpy(), two.cpu().numpy(), ts.cpu().numpy())


@pytest.mark.parametrize("B,H,S,k", [(1, 64, 40000, 2048), (5, 64, 7000, 512), (8, 64, 128, 64),
                                     (2, 64, 75000, 100), (16, 64, 32768, 1024), (2, 64, 129, 2048),
                                     (3, 40, 20000, 100), (4, 64, 300, 1), (20, 64, 5000, 256),
                                     (600, 64, 2048, 512), (161, 64, 3001, 2048), (600, 24, 1000, 100), (601, 64, 777, 2048),
                                     (1, 64, 131072, 2048)])
def test_fused_shapes(cuda_device, B, H, S, k):
    # whole-row groups (B >= 148 groups' worth of work, short rows) and split
    # rows; ragged S, rows longer than one CTA's 16-bit counters (S = 131072:
    # 1024 tiles over several CTAs), valid_len of 0, negative or past S
    q, kc, w = inputs.indexer_factors(seed=B * 5 + S + H, batch=B, n=S, heads=H)
    g = np.random.default_rng(S + B)
    vl = g.integers(-3, S + 5, size=B).astype(np.int32)
    vl[0] = S
    if B > 1:
        vl[1] = 0
    qd, kd, wd, vd = dev_inputs(q, kc, w, vl)
    idx, score = ds.ds_indexer_topk(qd, kd, wd, k, valid_len=vd, return_score=True)
    torch.cuda.synchronize()
    assert ds.ds_get_device_status() == ds.DS_OK
    check_selection(q, kc, w, vl, k, idx.cpu().numpy(), score.cpu().numpy())


@pytest.mark.parametrize("B,H,S,k", [(8, 64, 32768, 2048), (3, 64, 5000, 1000), (2, 24, 777, 700),
                                     (640, 64, 1000, 300), (160, 16, 2000, 2048), (600, 16, 300, 50)])
def test_fused_exact_arithmetic(cuda_device, B, H, S, k):
    # small-integer inputs: exact float32 scores with many equal values, so the
    # index sets must match the oracle's exactly, ties to the lower position
    q, kc, w = exact_inputs(B * 13 + S, B, H, S)
    qd, kd, wd, _ = dev_inputs(q, kc, w, None)
    idx, score = ds.ds_indexer_topk(qd, kd, wd, k, return_score=True)
    torch.cuda.synchronize()
    assert ds.ds_get_device_status() == ds.DS_OK
    ref_idx, ref_scores = oracle.indexer_topk(q, kc, w, k)
    idx, score = idx.cpu().numpy(), score.cpu().numpy()
    for t in range(B):
        m = int((ref_idx[t] >= 0).sum())
        assert np.array_equal(np.sort(idx[t, :m]), np.sort(ref_idx[t, :m])), f"row {t}"
        assert np.array_equal(score[t, :m].astype(np.float64), ref_scores[t, idx[t, :m]])


@pytest.mark.parametrize("B,S,L", [(2, 32768, 32768), (2, 20000, 12000), (2, 4096, 4000), (600, 2000, 2000)])
def test_fused_all_scores_equal(cuda_device, B, S, L):
    # zero weights: every score is 0, the whole row sits in one histogram bin
    # (past the candidate list's capacity for the longest rows) and the k lowest
    # positions must be returned
    q, kc, w = inputs.indexer_factors(seed=S, batch=B, n=S, heads=64)
    w = np.zeros_like(w)
    vl = np.full(B, L, dtype=np.int32)
    vl[1] = L // 3
    qd, kd, wd, vd = dev_inputs(q, kc, w, vl)
    idx, score = ds.ds_indexer_topk(qd, kd, wd, 2048, valid_len=vd, return_score=True)
    torch.cuda.synchronize()
    assert ds.ds_get_device_status() == ds.DS_OK
    idx = idx.cpu().numpy()
    for t in range(B):
        m = min(2048, int(vl[t]))
        assert np.array_equal(np.sort(idx[t, :m]), np.arange(m)), f"row {t}"
        assert np.all(idx[t, m:] == -1)
    assert np.all(score.cpu().numpy()[1, :min(2048, L // 3)] == 0.0)


@pytest.mark.parametrize("cluster", ["1", "2", "4", "8", "16"])
def test_split_row_selection_every_cluster_size(cuda_device, cluster, monkeypatch):
    # the split-row selection with its cluster capped (DS_HS_CLUSTER, a tuning
    # knob): every size must give the oracle's selection, sorted or not
    monkeypatch.setenv("DS_HS_CLUSTER", cluster)
    q, kc, w, vl = inputs.decode(seed=57, batch=8, S=32768, vl_lo=4096, vl_hi=32768)
    qd, kd, wd, vd = dev_inputs(q, kc, w, vl)
    idx, score = ds.ds_indexer_topk(qd, kd, wd, 1024, valid_len=vd, return_score=True)
    torch.cuda.synchronize()
    assert ds.ds_get_device_status() == ds.DS_OK
    check_selection(q, kc, w, vl, 1024, idx.cpu().numpy(), score.cpu().numpy())
    sidx, _ = ds.ds_indexer_topk_ex(qd, kd, wd, 1024, valid_len=vd, sorted_index=True)
    torch.cuda.synchronize()
    si = sidx.cpu().numpy()
    for t in range(8):
        m = int((si[t] >= 0).sum())
        assert np.all(np.diff(si[t, :m]) > 0), f"row {t}: not ascending"
        assert np.array_equal(si[t, :m], np.sort(idx.cpu().numpy()[t, :m])), f"row {t}: sorted set differs"


@pytest.mark.parametrize("B", [8, 600])
def test_fused_graph_replay(cuda_device, B):
    # the split-row path leaves its histograms and tickets zero for the next
    # launch; replaying a graph of 3 calls several times must keep results right
    q, kc, w, vl = inputs.decode(seed=43, batch=B, S=8192, vl_lo=1000, vl_hi=8192)
    qd, kd, wd, vd = dev_inputs(q, kc, w, vl)
    outs = [torch.empty((B, 512), dtype=torch.int32, device="cuda") for _ in range(3)]
    ds.ds_indexer_topk(qd, kd, wd, 512, valid_len=vd, out_idx=outs[0])   # warm-up outside capture
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for o in outs:
            ds.ds_indexer_topk(qd, kd, wd, 512, valid_len=vd, out_idx=o)
    for _ in range(3):
        for o in outs:
            o.fill_(-7)
        gr.replay()
        torch.cuda.synchronize()
        assert ds.ds_get_device_status() == ds.DS_OK
        for o in outs:
            check_selection(q, kc, w, vl, 512, o.cpu().numpy(), None)


# ---------------------------------------------------------------- per-row key caches, sorted output

def _per_row_case(seed, B, H, S):
    g = np.random.default_rng(seed)
    q, _, w = inputs.indexer_factors(seed=seed, batch=B, n=S, heads=H, d=128)
    kc3 = np.stack([inputs.indexer_factors(seed=seed + 100 + b, batch=1, n=S, heads=1, d=128)[1] for b in range(B)])
    vl = g.integers(1, S, size=B, endpoint=True).astype(np.int32)
    return q, kc3, w, vl


@pytest.mark.parametrize("B,H,S,k", [(4, 64, 2000, 300), (3, 32, 700, 128), (3, 16, 700, 64), (2, 8, 500, 33),
                                     (1, 64, 4096, 2048)])
def test_per_row_key_caches(cuda_device, B, H, S, k):
    q, kc3, w, vl = _per_row_case(40 + H, B, H, S)
    qd, kd, wd, vd = dev_inputs(q, kc3, w, vl)
    idx, score = ds.ds_indexer_topk_ex(qd, kd, wd, k, valid_len=vd, return_score=True)
    torch.cuda.synchronize()
    assert ds.ds_get_device_status() == ds.DS_OK
    check_selection(q, kc3, w, vl, k, idx.cpu().numpy(), score.cpu().numpy())


def test_per_row_exact_arithmetic_selects_exactly(cuda_device):
    # small integer q and keys, power-of-two w: every float32 sum is exact, so the
    # selected sets equal the oracle's (ties to the lower position)
    g = np.random.default_rng(77)
    B, H, S, k = 3, 64, 900, 100
    q = inputs.f32_to_bf16_bits(g.integers(-2, 3, (B, H, 128)).astype(np.float32))
    kc3 = inputs.f32_to_bf16_bits(g.integers(-2, 3, (B, S, 128)).astype(np.float32))
    w = (2.0 ** g.integers(-3, 3, (B, H))).astype(np.float32)
    vl = np.array([900, 450, 1], dtype=np.int32)
    qd, kd, wd, vd = dev_inputs(q, kc3, w, vl)
    idx, _ = ds.ds_indexer_topk_ex(qd, kd, wd, k, valid_len=vd)
    torch.cuda.synchronize()
    ref, _ = oracle.indexer_topk(q, kc3, w, k, vl)
    got = idx.cpu().numpy()
    for t in range(B):
        m = int((ref[t] >= 0).sum())
        assert sorted(got[t, :m].tolist()) == sorted(ref[t, :m].tolist())
        assert np.all(got[t, m:] == -1)


def test_ex_with_one_cache_matches_ds_indexer_topk(cuda_device):
    q, kc, w, vl = inputs.decode(seed=51, batch=8, S=8192, vl_lo=1000, vl_hi=8192)
    qd, kd, wd, vd = dev_inputs(q, kc, w, vl)
    a, _ = ds.ds_indexer_topk(qd, kd, wd, 1024, valid_len=vd)
    b, _ = ds.ds_indexer_topk_ex(qd, kd, wd, 1024, valid_len=vd)
    torch.cuda.synchronize()
    assert torch.equal(torch.sort(a, dim=1).values, torch.sort(b, dim=1).values)


@pytest.mark.parametrize("per_row", [False, True], ids=["one-cache", "per-row"])
def test_sorted_index_in_the_fused_path(cuda_device, per_row):
    if per_row:
        q, kc, w, vl = _per_row_case(61, 4, 64, 3000)
    else:
        q, kc, w, vl = inputs.decode(seed=62, batch=4, S=3000, vl_lo=100, vl_hi=3000)
    qd, kd, wd, vd = dev_inputs(q, kc, w, vl)
    u, su = ds.ds_indexer_topk_ex(qd, kd, wd, 512, valid_len=vd, return_score=True)
    s, ss = ds.ds_indexer_topk_ex(qd, kd, wd, 512, valid_len=vd, sorted_index=True, return_score=True)
    torch.cuda.synchronize()
    u, su, s, ss = u.cpu().numpy(), su.cpu().numpy(), s.cpu().numpy(), ss.cpu().numpy()
    for t in range(4):
        m = int((u[t] >= 0).sum())
        assert np.all(np.diff(s[t, :m]) > 0), "not in ascending position order"
        assert sorted(u[t, :m].tolist()) == s[t, :m].tolist()
        order = np.argsort(u[t, :m])
        assert np.array_equal(su[t, :m][order], ss[t, :m]), "scores do not follow their positions"
    check_selection(q, kc, w, vl, 512, s, ss)


def test_cache_stride_larger_than_S(cuda_device):
    # caches padded with 37 extra rows each, addressed through the stride
    B, H, S, k = 3, 64, 1200, 200
    q, kc3, w, vl = _per_row_case(71, B, H, S)
    padded = np.zeros((B, S + 37, 128), dtype=np.uint16)
    padded[:, :S] = kc3
    padded[:, S:] = inputs.f32_to_bf16_bits(np.full((B, 37, 128), 30.0, dtype=np.float32))  # would win if read
    qd, kd, wd, vd = dev_inputs(q, padded, w, vl)
    idx = torch.empty((B, k), dtype=torch.int32, device=cuda_device)
    from sparse_attention_top_ds_b200._native import load, _ptr, _stream_ptr
    rc = load().ds_indexer_topk_ex(_ptr(qd), _ptr(kd), S + 37, _ptr(wd), B, H, 128, S, _ptr(vd), k, 0,
                                   _ptr(idx), None, _stream_ptr(None))
    assert rc == ds.DS_OK
    torch.cuda.synchronize()
    check_selection(q, kc3, w, vl, k, idx.cpu().numpy(), None)
