"""Helpers shared by the GPU parity tests: host <-> device conversions and the
comparison rules.  Inputs come from sparse_attention_top_ds_b200.inputs, expected
values from the oracle; nothing here computes a selection."""

import numpy as np
import torch


def bf16_to_device(bits, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def f32_to_device(x, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def i32_to_device(x, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).to(device)


def bits_of(t):
    """Raw bit patterns of a CUDA bf16 / f32 tensor as a numpy uint16 / uint32 array."""
    if t.dtype == torch.bfloat16:
        return t.cpu().view(torch.int16).numpy().view(np.uint16)
    return t.cpu().numpy().view(np.uint32)


def assert_topk_exact(idx_gpu, val_gpu, raw, idx_ref, k, sorted_index):
    """Bit-exact parity of a top-k result with the oracle.

    idx_gpu / idx_ref are [batch, k]; the selected sets must be identical (the
    oracle's tie rule makes the set unique), padding identical, and each
    returned value the stored bit pattern of its position.
    """
    idx_gpu = np.asarray(idx_gpu).astype(np.int64)
    for t in range(idx_ref.shape[0]):
        ref = idx_ref[t]
        m = int((ref >= 0).sum())
        got = idx_gpu[t]
        assert int((got >= 0).sum()) == m, f"row {t}: {int((got >= 0).sum())} selected, expected {m}"
        assert np.all(got[m:] == -1), f"row {t}: padding"
        sel = got[:m]
        if sorted_index:
            assert np.all(np.diff(sel) > 0), f"row {t}: not in ascending order"
        exp = np.sort(ref[:m])
        if not np.array_equal(np.sort(sel), exp):
            missing = np.setdiff1d(exp, sel)[:10]
            extra = np.setdiff1d(sel, exp)[:10]
            raise AssertionError(f"row {t}: index sets differ; missing {missing}, extra {extra}")
        if val_gpu is not None:
            vals = val_gpu[t]
            assert np.array_equal(vals[:m], raw[t][sel]), f"row {t}: values are not the stored bits"
