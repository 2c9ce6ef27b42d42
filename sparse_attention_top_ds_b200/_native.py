"""ctypes binding of libdstopk.so: argument marshalling only.

Every step of the selection runs in the library's CUDA kernels.  If the shared
library is missing or cannot be loaded, every call raises; there is no
fallback implementation.
"""

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
# DS_TOPK_LIB may name another build, such as libdstopk_debug.so (device range checks)
_LIB_PATH = os.environ.get("DS_TOPK_LIB", os.path.join(_PKG, "libdstopk.so"))
DEBUG_LIB_PATH = os.path.join(_PKG, "libdstopk_debug.so")

DS_F32 = 0
DS_BF16 = 1

DS_OK = 0
DS_ERR_ARG = -1
DS_ERR_CUDA = -2
DS_ERR_TIMEOUT = -3
DS_ERR_UNSUPPORTED = -4
DS_ERR_NOMEM = -5
DS_ERR_RANGE = -6

DS_MAX_K = 2048
DS_INDEXER_DIM = 128
DS_INDEXER_MAX_HEADS = 64
DS_ATTN_MAX_DIM = 512
DS_ATTN_MAX_WINDOW = 4096
DS_ATTN_MAX_HEADS = 4096

_lib = None


class DsError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {strerror(code) if _lib is not None else code}")


def lib_path():
    return _LIB_PATH


def load():
    """Load the shared library once; raise if it is not there."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(
            f"libdstopk.so not found at {_LIB_PATH}; build it with "
            "`python -m sparse_attention_top_ds_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, i32p = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
    lib.ds_topk.argtypes = [vp, i32, i32, i32, i32, i32p, vp, vp, i32, i32, vp]
    lib.ds_topk.restype = i32
    lib.ds_indexer_score.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32p, vp, vp]
    lib.ds_indexer_score.restype = i32
    lib.ds_indexer_topk.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32p, i32, vp, vp, vp]
    lib.ds_indexer_topk.restype = i32
    lib.ds_indexer_topk_noalloc.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32p, i32, vp, vp, vp]
    lib.ds_indexer_topk_noalloc.restype = i32
    lib.ds_sparse_attention.argtypes = [vp, vp, ctypes.c_int64, i32, i32p, i32, vp, i32, i32p, vp,
                                        i32, i32, i32, ctypes.c_float, vp, vp, vp]
    lib.ds_sparse_attention.restype = i32
    lib.ds_indexer_topk_ex.argtypes = [vp, vp, ctypes.c_int64, vp, i32, i32, i32, i32, i32p, i32, i32, vp, vp, vp]
    lib.ds_indexer_topk_ex.restype = i32
    lib.ds_compress_fold.argtypes = [vp, i32, i32, ctypes.c_int64, vp, vp, ctypes.c_int64, vp]
    lib.ds_compress_fold.restype = i32
    lib.ds_indexer_qproj.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp]
    lib.ds_indexer_qproj.restype = i32
    lib.ds_get_device_status.argtypes = [vp]
    lib.ds_get_device_status.restype = i32
    lib.ds_strerror.argtypes = [i32]
    lib.ds_strerror.restype = ctypes.c_char_p
    lib.ds_release.argtypes = []
    lib.ds_release.restype = None
    lib.ds_set_wait_limit.argtypes = [ctypes.c_int64]
    lib.ds_set_wait_limit.restype = i32
    lib.ds_plant_wait_fault.argtypes = [i32]
    lib.ds_plant_wait_fault.restype = i32
    lib.ds_debug_build.argtypes = []
    lib.ds_debug_build.restype = i32
    lib.ds_debug_stash_stamps.argtypes = [vp, i32]
    lib.ds_debug_stash_stamps.restype = i32
    lib.ds_read_floor.argtypes = [vp, ctypes.c_int64, i32, vp]
    lib.ds_read_floor.restype = i32
    _lib = lib
    return lib


def strerror(code):
    return load().ds_strerror(int(code)).decode()


def _check(code, where):
    if code != DS_OK:
        raise DsError(code, where)


# ------------------------------------------------------------------ raw pointer calls (C ABI)

def ds_topk_raw(scores, batch, n, k, dtype, valid_len, out_idx, out_val, return_value, sorted_index, stream):
    return load().ds_topk(scores, batch, n, k, dtype, valid_len, out_idx, out_val,
                          int(return_value), int(sorted_index), stream)


def ds_indexer_score_raw(q, kcache, w, batch, heads, d, S, valid_len, out_score, stream):
    return load().ds_indexer_score(q, kcache, w, batch, heads, d, S, valid_len, out_score, stream)


def ds_indexer_topk_raw(q, kcache, w, batch, heads, d, S, valid_len, k, out_idx, out_score, stream):
    return load().ds_indexer_topk(q, kcache, w, batch, heads, d, S, valid_len, k, out_idx, out_score, stream)


def ds_indexer_topk_noalloc_raw(q, kcache, w, batch, heads, d, S, valid_len, k, out_idx, out_score, stream):
    """The allocation-free variant (score rows in the library's fixed array)."""
    return load().ds_indexer_topk_noalloc(q, kcache, w, batch, heads, d, S, valid_len, k, out_idx, out_score,
                                          stream)


def ds_sparse_attention_raw(q, kv, kv_batch_stride, T, idx, k, win, W, win_len, sink, batch, heads, d, scale,
                            out, lse, stream):
    return load().ds_sparse_attention(q, kv, int(kv_batch_stride), T, idx, k, win, W, win_len, sink,
                                      batch, heads, d, float(scale), out, lse, stream)


def ds_indexer_qproj_raw(x, wq, ww, T, d_in, heads, d, q_out, w_out, stream):
    return load().ds_indexer_qproj(x, wq, ww, T, d_in, heads, d, q_out, w_out, stream)


def ds_get_device_status(stream=None):
    return load().ds_get_device_status(_stream_ptr(stream))


def ds_release():
    load().ds_release()


def ds_set_wait_limit(ns):
    """Limit of the kernels' bounded waits in ns (0: the default of one second)."""
    _check(load().ds_set_wait_limit(int(ns)), "ds_set_wait_limit")


def ds_plant_wait_fault(launches):
    """Testing the failure detection: the next `launches` scorer launches each
    make one of their bounded waits run out (DS_ERR_TIMEOUT in the status)."""
    _check(load().ds_plant_wait_fault(int(launches)), "ds_plant_wait_fault")


def ds_debug_build():
    """True for the DS_DEBUG build (device range checks -> DS_ERR_RANGE)."""
    return bool(load().ds_debug_build())


def ds_debug_stash_stamps(ctas):
    """DS_DEBUG build: the stash top-k kernel's phase stamps (ns), [ctas, 10] uint64."""
    import numpy as np
    out = np.zeros((ctas, 10), dtype=np.uint64)
    _check(load().ds_debug_stash_stamps(ctypes.c_void_p(out.ctypes.data), int(ctas)), "ds_debug_stash_stamps")
    return out


def ds_read_floor(x, ctas, stream=None):
    """Enqueue a read-only pass over the CUDA tensor x (its bytes split over ctas CTAs)."""
    _check(load().ds_read_floor(_ptr(x), x.numel() * x.element_size(), int(ctas), _stream_ptr(stream)),
           "ds_read_floor")


# ------------------------------------------------------------------ torch-tensor front end

def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _require(t, dtype, name, device=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def ds_topk(scores, k, valid_len=None, return_value=True, sorted_index=False,
            out_idx=None, out_val=None, stream=None):
    """Top-k of every row of a [batch, n] float32 / bfloat16 CUDA tensor.

    Returns (idx int32 [batch, k], val [batch, k] or None).  Without
    ``sorted_index`` the order of a row's selection is unspecified.
    """
    import torch
    if scores.dtype == torch.float32:
        dt = DS_F32
    elif scores.dtype == torch.bfloat16:
        dt = DS_BF16
    else:
        raise TypeError("scores must be float32 or bfloat16")
    _require(scores, None, "scores")
    if scores.dim() != 2:
        raise ValueError("scores must be [batch, n]")
    batch, n = scores.shape
    dev = scores.device
    if valid_len is not None:
        _require(valid_len, torch.int32, "valid_len", dev)
    if out_idx is None:
        out_idx = torch.empty((batch, k), dtype=torch.int32, device=dev)
    _require(out_idx, torch.int32, "out_idx", dev)
    if return_value and out_val is None:
        out_val = torch.empty((batch, k), dtype=scores.dtype, device=dev)
    with torch.cuda.device(dev):
        rc = ds_topk_raw(_ptr(scores), batch, n, k, dt, _ptr(valid_len), _ptr(out_idx),
                         _ptr(out_val) if return_value else None, return_value, sorted_index,
                         _stream_ptr(stream))
    _check(rc, "ds_topk")
    return out_idx, (out_val if return_value else None)


def _indexer_args(q, kcache, w, valid_len):
    import torch
    _require(q, torch.bfloat16, "q")
    dev = q.device
    _require(kcache, torch.bfloat16, "kcache", dev)
    _require(w, torch.float32, "w", dev)
    if q.dim() != 3 or kcache.dim() != 2 or w.dim() != 2:
        raise ValueError("q [batch,heads,d], kcache [S,d], w [batch,heads]")
    batch, heads, d = q.shape
    S = kcache.shape[0]
    if kcache.shape[1] != d or tuple(w.shape) != (batch, heads):
        raise ValueError("shape mismatch between q, kcache and w")
    if valid_len is not None:
        _require(valid_len, torch.int32, "valid_len", dev)
    return dev, batch, heads, d, S


def ds_indexer_score(q, kcache, w, valid_len=None, out=None, stream=None):
    """Indexer score rows [batch, S] float32 (-inf at positions >= valid_len)."""
    import torch
    dev, batch, heads, d, S = _indexer_args(q, kcache, w, valid_len)
    if out is None:
        out = torch.empty((batch, S), dtype=torch.float32, device=dev)
    _require(out, torch.float32, "out", dev)
    with torch.cuda.device(dev):
        rc = ds_indexer_score_raw(_ptr(q), _ptr(kcache), _ptr(w), batch, heads, d, S,
                                  _ptr(valid_len), _ptr(out), _stream_ptr(stream))
    _check(rc, "ds_indexer_score")
    return out


def ds_indexer_topk(q, kcache, w, k, valid_len=None, return_score=False,
                    out_idx=None, out_score=None, stream=None):
    """Top-k positions of every indexer score row: (idx int32 [batch,k], score f32 [batch,k] or None)."""
    import torch
    dev, batch, heads, d, S = _indexer_args(q, kcache, w, valid_len)
    if out_idx is None:
        out_idx = torch.empty((batch, k), dtype=torch.int32, device=dev)
    _require(out_idx, torch.int32, "out_idx", dev)
    if return_score and out_score is None:
        out_score = torch.empty((batch, k), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        rc = ds_indexer_topk_raw(_ptr(q), _ptr(kcache), _ptr(w), batch, heads, d, S,
                                 _ptr(valid_len), k, _ptr(out_idx),
                                 _ptr(out_score) if return_score else None, _stream_ptr(stream))
    _check(rc, "ds_indexer_topk")
    return out_idx, (out_score if return_score else None)


def ds_indexer_topk_noalloc(q, kcache, w, k, valid_len=None, return_score=False,
                            out_idx=None, out_score=None, stream=None):
    """ds_indexer_topk through the allocation-free entry point (batch * S <= 262144)."""
    import torch
    dev, batch, heads, d, S = _indexer_args(q, kcache, w, valid_len)
    if out_idx is None:
        out_idx = torch.empty((batch, k), dtype=torch.int32, device=dev)
    _require(out_idx, torch.int32, "out_idx", dev)
    if return_score and out_score is None:
        out_score = torch.empty((batch, k), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        rc = ds_indexer_topk_noalloc_raw(_ptr(q), _ptr(kcache), _ptr(w), batch, heads, d, S,
                                         _ptr(valid_len), k, _ptr(out_idx),
                                         _ptr(out_score) if return_score else None, _stream_ptr(stream))
    _check(rc, "ds_indexer_topk_noalloc")
    return out_idx, (out_score if return_score else None)


def ds_sparse_attention(q, kv, idx, scale=None, win=None, win_len=None, sink=None, return_lse=False,
                        out=None, lse=None, stream=None):
    """Multi-query attention of every query head over the selected cache rows
    plus a sliding window.

    q    bf16 [batch, heads, d];  kv  bf16 [T, d] (one cache for every batch
    row) or [batch, T, d];  idx  int32 [batch, k] or None (window only);
    win  bf16 [batch, W, d] or None;  win_len  int32 [batch] or None (= W);
    sink float32 [heads] or None;  scale  default 1/sqrt(d).
    Returns out bf16 [batch, heads, d], or (out, lse float32 [batch, heads]).
    """
    import math
    import torch
    _require(q, torch.bfloat16, "q")
    dev = q.device
    _require(kv, torch.bfloat16, "kv", dev)
    if q.dim() != 3:
        raise ValueError("q must be [batch, heads, d]")
    batch, heads, d = q.shape
    if kv.dim() == 2:
        T, stride = kv.shape[0], 0
    elif kv.dim() == 3 and kv.shape[0] == batch:
        T, stride = kv.shape[1], kv.shape[1]
    else:
        raise ValueError("kv must be [T, d] or [batch, T, d]")
    if kv.shape[-1] != d:
        raise ValueError("kv and q differ in d")
    k = 0
    if idx is not None:
        _require(idx, torch.int32, "idx", dev)
        if idx.dim() != 2 or idx.shape[0] != batch:
            raise ValueError("idx must be [batch, k]")
        k = idx.shape[1]
    W = 0
    if win is not None:
        _require(win, torch.bfloat16, "win", dev)
        if win.dim() != 3 or win.shape[0] != batch or win.shape[2] != d:
            raise ValueError("win must be [batch, W, d]")
        W = win.shape[1]
    if win_len is not None:
        _require(win_len, torch.int32, "win_len", dev)
    if sink is not None:
        _require(sink, torch.float32, "sink", dev)
        if sink.numel() != heads:
            raise ValueError("sink must hold one logit per head")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((batch, heads, d), dtype=torch.bfloat16, device=dev)
    _require(out, torch.bfloat16, "out", dev)
    if return_lse and lse is None:
        lse = torch.empty((batch, heads), dtype=torch.float32, device=dev)
    if lse is not None:
        _require(lse, torch.float32, "lse", dev)
    with torch.cuda.device(dev):
        rc = ds_sparse_attention_raw(_ptr(q), _ptr(kv), stride, T, _ptr(idx), k, _ptr(win), W, _ptr(win_len),
                                     _ptr(sink), batch, heads, d, scale, _ptr(out), _ptr(lse),
                                     _stream_ptr(stream))
    _check(rc, "ds_sparse_attention")
    return (out, lse) if return_lse else out


def ds_indexer_qproj(x, wq, ww=None, heads=None, q_out=None, w_out=None, stream=None):
    """Indexer queries and per-head weights from one input row per token.

    x bf16 [T, d_in];  wq bf16 [heads * 128, d_in];  ww bf16 [heads, d_in] or None.
    Returns (q bf16 [T, heads, 128], w float32 [T, heads] or None).
    """
    import torch
    _require(x, torch.bfloat16, "x")
    dev = x.device
    _require(wq, torch.bfloat16, "wq", dev)
    if x.dim() != 2 or wq.dim() != 2 or wq.shape[1] != x.shape[1] or wq.shape[0] % DS_INDEXER_DIM:
        raise ValueError("x [T, d_in], wq [heads * 128, d_in]")
    T, d_in = x.shape
    H = wq.shape[0] // DS_INDEXER_DIM if heads is None else int(heads)
    if ww is not None:
        _require(ww, torch.bfloat16, "ww", dev)
        if tuple(ww.shape) != (H, d_in):
            raise ValueError("ww must be [heads, d_in]")
    if q_out is None:
        q_out = torch.empty((T, H, DS_INDEXER_DIM), dtype=torch.bfloat16, device=dev)
    _require(q_out, torch.bfloat16, "q_out", dev)
    if ww is not None and w_out is None:
        w_out = torch.empty((T, H), dtype=torch.float32, device=dev)
    if w_out is not None:
        _require(w_out, torch.float32, "w_out", dev)
    with torch.cuda.device(dev):
        rc = ds_indexer_qproj_raw(_ptr(x), _ptr(wq), _ptr(ww), T, d_in, H, DS_INDEXER_DIM, _ptr(q_out),
                                  _ptr(w_out) if ww is not None else None, _stream_ptr(stream))
    _check(rc, "ds_indexer_qproj")
    return q_out, (w_out if ww is not None else None)


def ds_indexer_topk_ex(q, kcache, w, k, valid_len=None, sorted_index=False, return_score=False,
                       out_idx=None, out_score=None, stream=None):
    """ds_indexer_topk with kcache [S, d] (shared) or [batch, S, d] (one cache per
    row), and optional position-sorted output."""
    import torch
    _require(q, torch.bfloat16, "q")
    dev = q.device
    _require(kcache, torch.bfloat16, "kcache", dev)
    _require(w, torch.float32, "w", dev)
    batch, heads, d = q.shape
    if kcache.dim() == 2:
        S, stride = kcache.shape[0], 0
    elif kcache.dim() == 3 and kcache.shape[0] == batch:
        S, stride = kcache.shape[1], kcache.shape[1]
    else:
        raise ValueError("kcache must be [S, d] or [batch, S, d]")
    if kcache.shape[-1] != d or tuple(w.shape) != (batch, heads):
        raise ValueError("shape mismatch between q, kcache and w")
    if valid_len is not None:
        _require(valid_len, torch.int32, "valid_len", dev)
    if out_idx is None:
        out_idx = torch.empty((batch, k), dtype=torch.int32, device=dev)
    _require(out_idx, torch.int32, "out_idx", dev)
    if return_score and out_score is None:
        out_score = torch.empty((batch, k), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        rc = load().ds_indexer_topk_ex(_ptr(q), _ptr(kcache), int(stride), _ptr(w), batch, heads, d, S,
                                       _ptr(valid_len), k, int(bool(sorted_index)), _ptr(out_idx),
                                       _ptr(out_score) if return_score else None, _stream_ptr(stream))
    _check(rc, "ds_indexer_topk_ex")
    return out_idx, (out_score if return_score else None)


def ds_compress_fold(rows, gate, out=None, stream=None):
    """Fold each batch row's 4 rows into 1 (gated weighted sum).

    rows bf16 [batch, 4, D] (any batch stride, rows contiguous within a batch
    row); gate bf16 [D]; out bf16 [batch, D] or a strided [batch, D] view (for
    instance cache[:, j, :]).  Returns out.
    """
    import torch
    if not isinstance(rows, torch.Tensor) or rows.dtype != torch.bfloat16 or not rows.is_cuda:
        raise TypeError("rows must be a CUDA bfloat16 tensor")
    if rows.dim() != 3 or rows.shape[1] != 4 or rows.stride(2) != 1 or rows.stride(1) != rows.shape[2]:
        raise ValueError("rows must be [batch, 4, D] with contiguous rows")
    dev = rows.device
    batch, _, D = rows.shape
    _require(gate, torch.bfloat16, "gate", dev)
    if gate.numel() != D:
        raise ValueError("gate must hold D elements")
    if out is None:
        out = torch.empty((batch, D), dtype=torch.bfloat16, device=dev)
    if out.dtype != torch.bfloat16 or out.device != dev or out.dim() != 2 or out.stride(1) != 1 or out.shape[1] != D:
        raise ValueError("out must be a [batch, D] bfloat16 view with contiguous rows")
    with torch.cuda.device(dev):
        rc = load().ds_compress_fold(_ptr(rows), batch, D, rows.stride(0), _ptr(gate), _ptr(out), out.stride(0),
                                     _stream_ptr(stream))
    _check(rc, "ds_compress_fold")
    return out
