"""GPU parity of ds_compress_fold with the oracle (the stated reading of the
gate; the pages give none, so this parity is against that reading).

Bar: |out - ref| <= 2^-8 |ref| + 2^-14 max|x| (one bfloat16 rounding of the
output plus float32 scores and sums over at most 4096 channels).
"""

import numpy as np
import pytest
import torch

import sparse_attention_top_ds_b200 as ds
from oracle import compress_fold
from sparse_attention_top_ds_b200 import inputs

from gpu_util import bf16_to_device, bits_of

pytestmark = pytest.mark.gpu


def _dec(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _check(rows, gate, got):
    ref = compress_fold(rows, gate)
    xmax = np.abs(_dec(rows)).max(axis=(1, 2))[:, None]
    err = np.abs(got - ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 2.0 ** -14 * xmax), f"worst excess {np.max(err - 2.0 ** -8 * np.abs(ref))}"


@pytest.mark.parametrize("B,D,scale", [(8, 512, 1.0), (8, 128, 4.0), (3, 8, 1.0), (37, 4096, 2.0), (1, 1000, 30.0)])
def test_matches_oracle(cuda_device, B, D, scale):
    rows, gate = inputs.compress(seed=300 + D, batch=B, D=D, gate_scale=scale)
    out = ds.ds_compress_fold(bf16_to_device(rows, cuda_device), bf16_to_device(gate, cuda_device))
    torch.cuda.synchronize()
    _check(rows, gate, _dec(bits_of(out)))


def test_strided_rows_into_a_cache_position(cuda_device):
    # the last 4 rows of a [B, W, D] window, folded into position j of a [B, T, D] cache
    B, W, T, D, j = 4, 16, 10, 256, 7
    g = np.random.default_rng(8)
    win = inputs.f32_to_bf16_bits(g.standard_normal((B, W, D), dtype=np.float32))
    _, gate = inputs.compress(seed=9, batch=1, D=D)
    wd = bf16_to_device(win, cuda_device)
    cache = torch.zeros((B, T, D), dtype=torch.bfloat16, device=cuda_device)
    ds.ds_compress_fold(wd[:, W - 4:, :], bf16_to_device(gate, cuda_device), out=cache[:, j, :])
    torch.cuda.synchronize()
    got = _dec(bits_of(cache))
    _check(win[:, W - 4:, :], gate, got[:, j, :])
    others = np.delete(got, j, axis=1)
    assert np.all(others == 0.0), "rows other than position j were written"
