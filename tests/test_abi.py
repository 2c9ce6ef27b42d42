"""The C-ABI library builds, loads and exports every entry point that
include/ds_topk.h declares; host-side argument checks answer without a GPU;
the Python binding fails loudly when the library is missing (CPU only)."""

import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ds_topk.h")


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_top_ds_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def declared_entry_points():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ds_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for n in ("ds_topk", "ds_indexer_score", "ds_indexer_topk", "ds_indexer_topk_ex", "ds_indexer_qproj",
              "ds_compress_fold", "ds_sparse_attention", "ds_get_device_status", "ds_strerror", "ds_release"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_entry_points():
        assert hasattr(lib, name), f"{name} is declared but not exported"


def test_exported_symbols_have_c_linkage(lib):
    from sparse_attention_top_ds_b200 import build
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (ds_\w+)$", out, flags=re.M))
    assert set(declared_entry_points()) <= exported


@pytest.fixture(scope="module")
def debug_lib(lib):
    from sparse_attention_top_ds_b200 import build
    assert os.path.exists(build.LIB_DEBUG), "build() makes libdstopk_debug.so beside libdstopk.so"
    return ctypes.CDLL(build.LIB_DEBUG)


def test_debug_build_flag_plumbing(lib, debug_lib):
    # the DS_DEBUG compile flag reaches the device code's range checks: the
    # release library reports 0, the debug library 1, and both export the
    # same boundary with C linkage
    from sparse_attention_top_ds_b200 import build
    assert lib.ds_debug_build() == 0
    assert debug_lib.ds_debug_build() == 1
    for name in declared_entry_points():
        assert hasattr(debug_lib, name), f"{name} is not exported by the debug build"
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB_DEBUG], capture_output=True, text=True).stdout
    assert set(declared_entry_points()) <= set(re.findall(r"\bT (ds_\w+)$", out, flags=re.M))
    debug_lib.ds_strerror.restype = ctypes.c_char_p
    assert b"DS_ERR_RANGE" in debug_lib.ds_strerror(-6)


def test_debug_build_is_rebuilt_with_the_release_build():
    # the build compiles the debug library with -DDS_DEBUG and the release one without
    from sparse_attention_top_ds_b200 import build
    src = open(build.__file__).read()
    assert '"-DDS_DEBUG"' in src
    assert not build.stale(build.LIB) and not build.stale(build.LIB_DEBUG)


def test_wait_limit_and_planted_fault_arguments_need_no_gpu(lib):
    lib.ds_set_wait_limit.argtypes = [ctypes.c_int64]
    lib.ds_plant_wait_fault.argtypes = [ctypes.c_int]
    assert lib.ds_set_wait_limit(-1) == -1
    assert lib.ds_set_wait_limit(60_000_000_001) == -1
    assert lib.ds_set_wait_limit(1_000_000) == 0
    assert lib.ds_set_wait_limit(0) == 0
    assert lib.ds_plant_wait_fault(-1) == -1
    assert lib.ds_plant_wait_fault(0) == 0


def test_measurement_entry_points_need_no_gpu(lib, debug_lib):
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.ds_read_floor.argtypes = [vp, i64, ctypes.c_int, vp]
    assert lib.ds_read_floor(None, 1024, 8, None) == -1                  # null
    assert lib.ds_read_floor(vp(0x100008), 1024, 8, None) == -1          # not 16-byte aligned
    assert lib.ds_read_floor(vp(0x100000), 1000, 8, None) == -1          # not a multiple of 16
    assert lib.ds_read_floor(vp(0x100000), 1024, 0, None) == -1          # no CTA
    lib.ds_debug_stash_stamps.argtypes = [vp, ctypes.c_int]
    buf = (ctypes.c_uint64 * 10)()
    assert lib.ds_debug_stash_stamps(buf, 1) == -4                       # release build: unsupported
    debug_lib.ds_debug_stash_stamps.argtypes = [vp, ctypes.c_int]
    assert debug_lib.ds_debug_stash_stamps(None, 1) == -1
    assert debug_lib.ds_debug_stash_stamps(buf, 0) == -1
    assert debug_lib.ds_debug_stash_stamps(buf, 1025) == -1


def test_strerror(lib):
    lib.ds_strerror.restype = ctypes.c_char_p
    assert lib.ds_strerror(0) == b"DS_OK"
    assert b"argument" in lib.ds_strerror(-1)
    assert b"unknown" in lib.ds_strerror(12345)
    assert b"DS_ERR_RANGE" in lib.ds_strerror(-6)


def test_argument_errors_need_no_gpu(lib):
    # every one of these is rejected on the host before any CUDA call
    vp = ctypes.c_void_p
    fake = vp(0x100000)
    lib.ds_topk.restype = ctypes.c_int
    lib.ds_topk.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp,
                            ctypes.c_int, ctypes.c_int, vp]
    assert lib.ds_topk(None, 1, 10, 5, 0, None, fake, fake, 1, 0, None) == -1      # null scores
    assert lib.ds_topk(fake, 0, 10, 5, 0, None, fake, fake, 1, 0, None) == -1      # batch
    assert lib.ds_topk(fake, 1, 10, 0, 0, None, fake, fake, 1, 0, None) == -1      # k = 0
    assert lib.ds_topk(fake, 1, 10, 2049, 0, None, fake, fake, 1, 0, None) == -1   # k > max
    assert lib.ds_topk(fake, 1, 10, 5, 7, None, fake, fake, 1, 0, None) == -1      # dtype
    assert lib.ds_topk(fake, 1, 10, 5, 0, None, fake, None, 1, 0, None) == -1      # out_val missing
    assert lib.ds_topk(fake, 1, (1 << 24) + 1, 5, 0, None, fake, fake, 1, 0, None) == -1  # row too long
    assert lib.ds_topk(vp(0x100001), 1, 10, 5, 0, None, fake, fake, 1, 0, None) == -1  # misaligned
    lib.ds_indexer_topk.restype = ctypes.c_int
    lib.ds_indexer_topk.argtypes = [vp, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp,
                                    ctypes.c_int, vp, vp, vp]
    assert lib.ds_indexer_topk(fake, fake, fake, 1, 64, 64, 100, None, 10, fake, None, None) == -1   # d
    assert lib.ds_indexer_topk(fake, fake, fake, 1, 65, 128, 100, None, 10, fake, None, None) == -1  # heads
    assert lib.ds_indexer_topk(fake, fake, fake, 1, 64, 128, 100, None, 0, fake, None, None) == -1   # k
    assert lib.ds_indexer_topk(fake, vp(0x100008), fake, 1, 64, 128, 100, None, 10, fake, None, None) == -1


def test_attention_argument_errors_need_no_gpu(lib):
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f = lib.ds_sparse_attention
    f.restype = i32
    f.argtypes = [vp, vp, ctypes.c_int64, i32, vp, i32, vp, i32, vp, vp, i32, i32, i32, ctypes.c_float, vp, vp, vp]
    a = vp(0x100000)

    def call(q=a, kv=a, stride=0, T=100, idx=a, k=10, win=None, W=0, wl=None, sink=None, B=2, H=128, d=512,
             scale=0.04, out=a, lse=None):
        return f(q, kv, stride, T, idx, k, win, W, wl, sink, B, H, d, scale, out, lse, None)

    assert call(q=None) == -1
    assert call(kv=None) == -1
    assert call(out=None) == -1
    assert call(d=576) == -1                  # above the largest head_dim
    assert call(d=100) == -1                  # not a multiple of 64
    assert call(d=0) == -1
    assert call(T=0) == -1
    assert call(stride=-1) == -1
    assert call(k=2049) == -1
    assert call(k=-1) == -1
    assert call(idx=None) == -1               # k > 0 needs slots
    assert call(W=8) == -1                    # a window needs rows
    assert call(W=4097, win=a) == -1
    assert call(B=0) == -1
    assert call(B=65536) == -1
    assert call(H=0) == -1
    assert call(H=4097) == -1
    assert call(scale=float("nan")) == -1
    assert call(scale=float("inf")) == -1
    assert call(q=vp(0x100008)) == -1         # 16-byte alignment
    assert call(kv=vp(0x100004)) == -1
    assert call(out=vp(0x100002)) == -1
    assert call(W=8, win=vp(0x100008)) == -1
    assert call(lse=vp(0x100002)) == -1


def test_indexer_topk_ex_argument_errors_need_no_gpu(lib):
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f = lib.ds_indexer_topk_ex
    f.restype = i32
    f.argtypes = [vp, vp, ctypes.c_int64, vp, i32, i32, i32, i32, vp, i32, i32, vp, vp, vp]
    a = vp(0x100000)

    def call(stride=0, S=1000, k=100, sorted_index=0, d=128, H=64, q=a, idx=a):
        return f(q, a, stride, a, 2, H, d, S, None, k, sorted_index, idx, None, None)

    assert call(stride=-1) == -1
    assert call(stride=999) == -1          # shorter than a cache
    assert call(sorted_index=2) == -1
    assert call(k=0) == -1
    assert call(k=2049) == -1
    assert call(d=64) == -1
    assert call(H=65) == -1
    assert call(q=None) == -1
    assert call(idx=None) == -1
    assert call(S=(1 << 24) + 1, stride=0) == -1


def test_compress_argument_errors_need_no_gpu(lib):
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f = lib.ds_compress_fold
    f.restype = i32
    f.argtypes = [vp, i32, i32, ctypes.c_int64, vp, vp, ctypes.c_int64, vp]
    a = vp(0x100000)

    def call(rows=a, B=8, D=512, rs=2048, gate=a, out=a, os_=512):
        return f(rows, B, D, rs, gate, out, os_, None)

    assert call(rows=None) == -1
    assert call(gate=None) == -1
    assert call(out=None) == -1
    assert call(B=0) == -1
    assert call(D=4) == -1
    assert call(D=4104, rs=4 * 4104, os_=4104) == -1
    assert call(D=100) == -1              # not a multiple of 8
    assert call(rs=2047) == -1            # shorter than 4 rows
    assert call(rs=2052) == -1            # not a multiple of 8
    assert call(os_=511) == -1
    assert call(rows=vp(0x100008)) == -1  # 16-byte alignment
    assert call(out=vp(0x100004)) == -1


def test_qproj_argument_errors_need_no_gpu(lib):
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f = lib.ds_indexer_qproj
    f.restype = i32
    f.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp]
    a = vp(0x100000)

    def call(x=a, wq=a, ww=a, T=8, d_in=1536, H=64, d=128, q=a, w=a):
        return f(x, wq, ww, T, d_in, H, d, q, w, None)

    assert call(x=None) == -1
    assert call(wq=None) == -1
    assert call(q=None) == -1
    assert call(ww=None) == -1            # w_out without ww
    assert call(w=None) == -1             # ww without w_out
    assert call(T=0) == -1
    assert call(H=65) == -1
    assert call(H=0) == -1
    assert call(d=64) == -1
    assert call(d_in=1532) == -1          # not a multiple of 8
    assert call(d_in=8200) == -1
    assert call(d_in=0) == -1
    assert call(x=vp(0x100008)) == -1     # 16-byte alignment
    assert call(wq=vp(0x100004)) == -1
    assert call(q=vp(0x100001)) == -1
    assert call(w=vp(0x100002)) == -1


def test_binding_fails_loudly_without_the_library(tmp_path):
    code = ("import sparse_attention_top_ds_b200 as ds\n"
            "try:\n    ds.load()\nexcept RuntimeError as e:\n    print('RAISED', e)\n")
    env = dict(os.environ, DS_TOPK_LIB=str(tmp_path / "missing.so"), PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, cwd=ROOT)
    assert "RAISED" in out.stdout and "no CPU fallback" in out.stdout
