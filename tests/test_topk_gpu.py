"""GPU parity of ds_topk (through the C ABI) with the float64 oracle, on both
top-k kernels.

Bar: bit-exact index sets and value bit patterns, ties to the lower index.
Covers the standalone, sampling and indexer-style workloads at full size (the
oracle selects from the stored rows directly), the adversarial ascending rows,
and the edge cases: k = 1, k = n, k > n, valid_len below k / zero / negative /
above n, ragged and misaligned rows, constant rows, signed zeros, NaN and
infinities, tie boundaries that cross CTA slices, and every cluster size.
"""

import os

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_top_ds_b200 as ds
from sparse_attention_top_ds_b200 import inputs
from gpu_util import assert_topk_exact, bf16_to_device, f32_to_device, i32_to_device, bits_of

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=["cluster", "stash"])
def topk_kernel(request, monkeypatch):
    # ds_topk has two kernels (picked by the number of rows); every case runs
    # on both: the cluster-histogram kernel and the one-pass stash kernel
    monkeypatch.setenv("DS_TOPK_KERNEL", request.param)
    return request.param


def run_case(raw, dtype, k, valid_len=None, sorted_index=False, return_value=True):
    x = bf16_to_device(raw) if dtype == "bf16" else f32_to_device(raw.view(np.float32) if raw.dtype == np.uint32 else raw)
    vl = None if valid_len is None else i32_to_device(valid_len)
    idx, val = ds.ds_topk(x, k, valid_len=vl, return_value=return_value, sorted_index=sorted_index)
    torch.cuda.synchronize()
    assert ds.ds_get_device_status() == ds.DS_OK
    ref_idx, _ = oracle.topk_rows(raw, dtype, k, valid_len)
    rawbits = raw if dtype == "bf16" else (raw.view(np.uint32) if raw.dtype == np.float32 else raw)
    assert_topk_exact(idx.cpu().numpy(), bits_of(val) if return_value else None, rawbits, ref_idx, k, sorted_index)
    return idx


# ---------------------------------------------------------------- headline workloads

@pytest.mark.parametrize("sorted_index", [False, True])
def test_standalone_4x8192_bf16_k512(cuda_device, sorted_index):
    raw = inputs.standalone()
    run_case(raw, "bf16", 512, sorted_index=sorted_index)


@pytest.mark.parametrize("k", [64, 1024])
def test_sampling_64x129280_f32(cuda_device, k):
    x, planted = inputs.sampling()
    idx = run_case(x, "f32", k).cpu().numpy()
    for t in range(x.shape[0]):
        assert set(planted[t]).issubset(set(idx[t]))


_rows_cache = {}


def indexer_rows(n, batch=64):
    """Indexer-style bf16 rows: the oracle's float64 scores of seeded factors,
    rounded to float32 then bfloat16."""
    if n not in _rows_cache:
        q, keys, w = inputs.indexer_factors(seed=inputs.SEED_INDEXER + n, batch=batch, n=n)
        s = oracle.indexer_scores(q, keys, w)
        _rows_cache[n] = inputs.f32_to_bf16_bits(s.astype(np.float32))
    return _rows_cache[n]


@pytest.mark.parametrize("n", [32768, 131072])
@pytest.mark.parametrize("batch", [1, 8, 64])
@pytest.mark.parametrize("ascending", [False, True])
def test_indexer_style_bf16_k2048(cuda_device, n, batch, ascending):
    raw = indexer_rows(n)[:batch]
    if ascending:
        raw = inputs.sort_rows_ascending_bf16(raw)
    run_case(np.ascontiguousarray(raw), "bf16", 2048)


# ---------------------------------------------------------------- edge cases

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_k_one_and_k_equal_n_and_k_above_n(cuda_device, dtype):
    g = np.random.default_rng(0)
    x = g.standard_normal((5, 2048), dtype=np.float32)
    raw = inputs.f32_to_bf16_bits(x) if dtype == "bf16" else x
    run_case(raw, dtype, 1)
    run_case(raw, dtype, 2048)
    raw_small = raw[:, :1500].copy()
    run_case(raw_small, dtype, 2048)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_valid_len_variants(cuda_device, dtype):
    g = np.random.default_rng(1)
    x = g.standard_normal((7, 5000), dtype=np.float32)
    raw = inputs.f32_to_bf16_bits(x) if dtype == "bf16" else x
    vl = np.array([0, 1, 100, 5000, 7000, -5, 4095], dtype=np.int32)
    run_case(raw, dtype, 256, valid_len=vl)
    run_case(raw, dtype, 256, valid_len=vl, sorted_index=True, return_value=False)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n", [1, 7, 9, 1001, 8191, 33333, 129281])
def test_ragged_and_misaligned_rows(cuda_device, dtype, n):
    g = np.random.default_rng(n)
    x = g.standard_normal((3, n), dtype=np.float32)
    raw = inputs.f32_to_bf16_bits(x) if dtype == "bf16" else x
    for k in sorted({1, min(n, 37), min(n, 2048)}):
        run_case(raw, dtype, k)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_constant_rows_take_lowest_indices(cuda_device, dtype):
    x = np.full((2, 131072), 0.75, dtype=np.float32)
    raw = inputs.f32_to_bf16_bits(x) if dtype == "bf16" else x
    idx = run_case(raw, dtype, 2048).cpu().numpy()
    # without sorted_index the order of a row's selection is unspecified
    assert np.array_equal(np.sort(idx[0]), np.arange(2048))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_tie_boundary_crosses_slices(cuda_device, dtype):
    # values in {0, 1}: the selection is every 1 plus the lowest-index 0s, and
    # the 0s it needs lie in several CTA slices
    g = np.random.default_rng(3)
    x = (g.random((4, 131072)) < 0.01).astype(np.float32)
    raw = inputs.f32_to_bf16_bits(x) if dtype == "bf16" else x
    for k in (1500, 2048):
        run_case(raw, dtype, k)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_few_distinct_values(cuda_device, dtype):
    g = np.random.default_rng(4)
    x = g.choice(np.array([-1.0, 0.5, 2.0, 3.0, 7.0], dtype=np.float32), size=(6, 50000))
    raw = inputs.f32_to_bf16_bits(x) if dtype == "bf16" else x
    for k in (1, 100, 2047):
        run_case(raw, dtype, k)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_signed_zeros_nan_and_infinities(cuda_device, dtype):
    g = np.random.default_rng(5)
    x = g.standard_normal((3, 4000), dtype=np.float32)
    x[0, :] = 0.0
    x[0, ::3] = -0.0
    x[1, [10, 500, 3999]] = np.nan
    x[1, [11, 12]] = np.inf
    x[2, :] = -np.inf
    x[2, [7, 77]] = np.inf
    raw = inputs.f32_to_bf16_bits(x) if dtype == "bf16" else x
    if dtype == "bf16":
        raw[1, [10, 500, 3999]] = 0x7FC0          # quiet NaN
        raw[0, ::3] = 0x8000                      # -0
    for k in (1, 3, 5, 100, 2048):
        run_case(raw, dtype, k)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_thresholds_on_special_values(cuda_device, dtype):
    # long rows (the stash kernel streams them) whose k-th key is a NaN (more
    # NaNs of every payload and sign than k), a subnormal, a zero of either
    # sign, or -inf
    n = 40000
    g = np.random.default_rng(9)
    if dtype == "f32":
        nans = np.array([0x7FC00000, 0xFFC00000, 0x7F800001, 0xFFFFFFFF], dtype=np.uint32)
        sub = lambda m: g.integers(1, 0x007FFFFF, size=m, dtype=np.uint32)
        pz, nz, ninf, sign = 0x00000000, 0x80000000, 0xFF800000, 0x80000000
        raw = g.standard_normal((4, n), dtype=np.float32).view(np.uint32).copy()
    else:
        nans = np.array([0x7FC0, 0xFFC0, 0x7F81, 0xFFFF], dtype=np.uint16)
        sub = lambda m: g.integers(1, 0x007F, size=m, dtype=np.uint16)
        pz, nz, ninf, sign = 0x0000, 0x8000, 0xFF80, 0x8000
        raw = inputs.f32_to_bf16_bits(g.standard_normal((4, n), dtype=np.float32)).copy()
    raw[0, g.choice(n, 12000, replace=False)] = g.choice(nans, 12000)
    raw[1] = sub(n) | np.where(g.random(n) < 0.5, sign, 0).astype(raw.dtype)
    raw[1, g.choice(n, 3000, replace=False)] = pz
    raw[1, g.choice(n, 3000, replace=False)] = nz
    raw[2, :] = ninf
    raw[2, g.choice(n, 500, replace=False)] = raw[3, :500]
    raw[3, :] = np.where(g.random(n) < 0.5, pz, nz).astype(raw.dtype)
    raw[3, g.choice(n, 300, replace=False)] = sub(300) | sign
    for k in (100, 2048):
        run_case(raw, dtype, k)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ascending_and_descending(cuda_device, dtype):
    x = np.arange(100000, dtype=np.float32)[None, :].repeat(2, axis=0)
    x[1] = x[1][::-1]
    raw = inputs.f32_to_bf16_bits(x) if dtype == "bf16" else x
    run_case(raw, dtype, 2048)


def test_many_short_rows(cuda_device):
    g = np.random.default_rng(6)
    x = g.standard_normal((3000, 50), dtype=np.float32)
    run_case(x, "f32", 20)
    run_case(inputs.f32_to_bf16_bits(x), "bf16", 64)


def test_long_rows(cuda_device):
    g = np.random.default_rng(7)
    x = g.standard_normal((2, 1000003), dtype=np.float32)
    run_case(x, "f32", 2048)
    run_case(inputs.f32_to_bf16_bits(g.standard_normal((2, 2000001), dtype=np.float32)), "bf16", 2048)


@pytest.mark.parametrize("cluster", ["1", "2", "4", "8", "16"])
def test_every_cluster_size(cuda_device, cluster, monkeypatch):
    monkeypatch.setenv("DS_TOPK_CLUSTER", cluster)
    g = np.random.default_rng(8)
    x = g.standard_normal((3, 20000), dtype=np.float32)
    x[:, 5000:5100] = 2.5                          # a tie block
    run_case(x, "f32", 1024)
    run_case(inputs.f32_to_bf16_bits(x), "bf16", 1024)


def test_argument_errors(cuda_device):
    x = torch.zeros((2, 100), dtype=torch.float32, device="cuda")
    with pytest.raises(ds.DsError):
        ds.ds_topk(x, 0)
    with pytest.raises(ds.DsError):
        ds.ds_topk(x, ds.DS_MAX_K + 1)
    too_long = torch.zeros((1, (1 << 24) + 8), dtype=torch.float32, device="cuda")
    with pytest.raises(ds.DsError):
        ds.ds_topk(too_long, 10)


def test_scores_produced_by_the_previous_kernel(cuda_device):
    # ds_topk may start while the previous kernel on the stream finishes
    # (programmatic dependent launch); it must still read that kernel's
    # finished output: here the scores come from a PyTorch kernel launched
    # right before, and each call's selection is checked against the oracle
    g = torch.Generator(device="cuda").manual_seed(11)
    idx_out = torch.empty((64, 256), dtype=torch.int32, device="cuda")
    for it in range(4):
        base = torch.randn((64, 40000), device="cuda", generator=g)
        scores = base * 3.0 + float(it)          # the producing kernel
        idx, val = ds.ds_topk(scores, 256, out_idx=idx_out)
        torch.cuda.synchronize()
        assert ds.ds_get_device_status() == ds.DS_OK
        raw = scores.cpu().numpy()
        ref_idx, _ = oracle.topk_rows(raw, "f32", 256)
        assert_topk_exact(idx.cpu().numpy(), bits_of(val), raw.view(np.uint32), ref_idx, 256, False)
