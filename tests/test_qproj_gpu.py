"""GPU parity of ds_indexer_qproj with the float64 oracle.

Both kernels are covered: input widths that are a multiple of 64 run on the
tensor cores (TMA + tcgen05), the others on the CUDA cores.  The bar, from the
arithmetic: |q - q_ref| <= 2^-8 |q_ref| + 2^-18 sum_i |x_i w_i|
(one bfloat16 rounding plus float32 accumulation), |w - w_ref| <= 2^-18 sum_i |x_i w_i|;
bit-exact (q = bf16(q_ref), w = w_ref) where every partial sum is exact in float32.
"""

import numpy as np
import pytest
import torch

import sparse_attention_top_ds_b200 as ds
from oracle import qproj as oracle_qproj, round_bf16
from sparse_attention_top_ds_b200 import inputs

from gpu_util import bf16_to_device, bits_of

pytestmark = pytest.mark.gpu


def _dec(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _run(x, wq, ww, dev, heads):
    q, w = ds.ds_indexer_qproj(bf16_to_device(x, dev), bf16_to_device(wq, dev),
                               None if ww is None else bf16_to_device(ww, dev), heads=heads)
    torch.cuda.synchronize()
    return _dec(bits_of(q)), (None if w is None else w.cpu().numpy().astype(np.float64))


def _check(x, wq, ww, q, w, heads):
    qr, wr = oracle_qproj(x, wq, ww, heads=heads)
    xa, wqa = np.abs(_dec(x)), np.abs(_dec(wq))
    bound_q = (xa @ wqa.T).reshape(qr.shape)               # sum_i |x_i w_i| per output
    err = np.abs(q - qr)
    assert np.all(err <= 2.0 ** -8 * np.abs(qr) + 2.0 ** -18 * bound_q + 1e-30), \
        f"q: worst excess {np.max(err - 2.0 ** -8 * np.abs(qr) - 2.0 ** -18 * bound_q):.3e}"
    if ww is not None:
        bound_w = xa @ np.abs(_dec(ww)).T
        assert np.all(np.abs(w - wr) <= 2.0 ** -18 * bound_w + 1e-30)


CASES = [
    # T, d_in, heads, with_w
    (8, 1536, 64, True),     # the decode workload
    (1, 8, 1, False),
    (13, 136, 3, True),      # input width not a multiple of 256; two token groups, ragged
    (33, 4096, 64, True),    # five token groups
    (3, 8192, 2, True),      # the widest input
    (8, 1528, 64, False),
]


@pytest.mark.parametrize("case", CASES, ids=[f"T{c[0]}din{c[1]}H{c[2]}{'w' if c[3] else ''}" for c in CASES])
def test_matches_oracle(case, cuda_device):
    T, d_in, H, with_w = case
    x, wq, ww = inputs.qproj(seed=200 + T + d_in, T=T, d_in=d_in, heads=H, with_w=with_w)
    q, w = _run(x, wq, ww, cuda_device, H)
    _check(x, wq, ww, q, w, H)


@pytest.mark.parametrize("d_in", [256, 264], ids=["tensor-cores", "cuda-cores"])
def test_exact_arithmetic_is_bit_exact(d_in, cuda_device):
    # small integers: every product and partial sum is exact in float32, so the
    # only rounding is q's to bfloat16 (the oracle's round_bf16).  Widths that
    # are a multiple of 64 run on the tensor cores, the others on the CUDA cores.
    g = np.random.default_rng(5)
    T, H = 11, 4
    x = inputs.f32_to_bf16_bits(g.integers(-3, 4, (T, d_in)).astype(np.float32))
    wq = inputs.f32_to_bf16_bits(g.integers(-3, 4, (H * 128, d_in)).astype(np.float32) * np.float32(1.0 / 1024))
    ww = inputs.f32_to_bf16_bits(g.integers(-3, 4, (H, d_in)).astype(np.float32))
    q, w = _run(x, wq, ww, cuda_device, H)
    qr, wr = oracle_qproj(x, wq, ww, heads=H)
    assert np.array_equal(q, round_bf16(qr))
    assert np.array_equal(w, wr)


def test_feeds_the_indexer_on_one_stream(cuda_device):
    """The projection's outputs read by ds_indexer_topk right after it
    (programmatic dependent launch) give the same selection as when read after
    a synchronisation."""
    x, wq, ww = inputs.qproj(seed=9)
    _, kc, _, vl = inputs.decode(seed=10, S=8192, vl_lo=2000, vl_hi=8192)
    dev = cuda_device
    xd, wqd, wwd = bf16_to_device(x, dev), bf16_to_device(wq, dev), bf16_to_device(ww, dev)
    kcd = bf16_to_device(kc, dev)
    vld = torch.from_numpy(vl).to(dev)
    s = torch.cuda.Stream(dev)
    with torch.cuda.stream(s):
        for _ in range(3):
            q, w = ds.ds_indexer_qproj(xd, wqd, wwd)
            idx, _ = ds.ds_indexer_topk(q, kcd, w, 512, valid_len=vld)
    s.synchronize()
    q2, w2 = ds.ds_indexer_qproj(xd, wqd, wwd)
    torch.cuda.synchronize()
    idx2, _ = ds.ds_indexer_topk(q2.clone(), kcd, w2.clone(), 512, valid_len=vld)
    torch.cuda.synchronize()
    assert torch.equal(torch.sort(idx, dim=1).values, torch.sort(idx2, dim=1).values)
    assert ds.ds_get_device_status() == ds.DS_OK
