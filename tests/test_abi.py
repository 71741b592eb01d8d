"""CPU checks of the C-ABI library: it loads, exports every entry point the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from weight_only_int4_w4_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4.h")


@pytest.fixture(scope="module")
def lib():
    path = build.build_library()
    return ctypes.CDLL(path)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(w4[a-z0-9_]*)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("w4_quantize", "w4_pack", "w4a16_gemm", "w4a16_gemm_workspace_size", "w4_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def _setup(lib):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    lib.w4_quantize.argtypes = [P, ctypes.c_int, P, I64, I64, ctypes.c_int, P, P, P, P, P]
    lib.w4_pack.argtypes = [P, I64, I64, P, P]
    lib.w4a16_gemm.argtypes = [P, ctypes.c_int, I64, I64, I64, ctypes.c_int, P, P, P, P, P, ctypes.c_int, P,
                               ctypes.c_size_t, P]
    lib.w4a16_gemm_workspace_size.argtypes = [I64, I64, I64]
    lib.w4a16_gemm_workspace_size.restype = ctypes.c_size_t
    lib.w4_status_string.argtypes = [ctypes.c_int]
    lib.w4_status_string.restype = ctypes.c_char_p
    lib.w4_last_error.restype = ctypes.c_char_p


A = 0x10000  # fake, 16-byte aligned "device" addresses: never dereferenced (rejected first)


def test_status_strings(lib):
    _setup(lib)
    assert lib.w4_status_string(0) == b"W4_OK"
    assert lib.w4_status_string(1) == b"W4_ERR_INVALID_ARG"
    assert lib.w4_status_string(2) == b"W4_ERR_UNSUPPORTED"
    assert lib.w4_status_string(3) == b"W4_ERR_CUDA"


@pytest.mark.parametrize("N,K,group,expect", [
    (0, 128, 128, 1),      # empty
    (4, 0, 128, 1),
    (4, 200, 128, 1),      # K not a multiple of the group
    (4, 256, 48, 2),       # unsupported group size (32, 64 and 128 are served)
    (-1, 128, 128, 1),
])
def test_quantize_rejects_bad_shapes(lib, N, K, group, expect):
    _setup(lib)
    st = lib.w4_quantize(A, 0, None, N, K, group, A, A, A, None, None)
    assert st == expect, lib.w4_last_error()


def test_quantize_rejects_null_and_misaligned(lib):
    _setup(lib)
    assert lib.w4_quantize(None, 0, None, 4, 128, 128, A, A, A, None, None) == 1
    assert lib.w4_quantize(A, 0, None, 4, 128, 128, None, A, A, None, None) == 1
    assert lib.w4_quantize(A + 4, 0, None, 4, 128, 128, A, A, A, None, None) == 1
    assert lib.w4_quantize(A, 0, A + 8, 4, 128, 128, A, A, A, None, None) == 1
    assert lib.w4_quantize(A, 0, A + 8, 4, 128, 128, A, A, A, None, None) == 1
    assert b"aligned" in lib.w4_last_error()
    assert lib.w4_quantize(A, 7, None, 4, 128, 128, A, A, A, None, None) == 2  # unknown dtype


def test_pack_rejects(lib):
    _setup(lib)
    assert lib.w4_pack(A, 4, 48, A, None) == 1   # K not a multiple of 32
    assert lib.w4_pack(None, 4, 64, A, None) == 1
    assert lib.w4_pack(A, 4, 64, A + 1, None) == 1


def test_gemm_rejects(lib):
    _setup(lib)
    g = lambda **kw: lib.w4a16_gemm(kw.get("X", A), kw.get("xd", 2), kw.get("M", 1), kw.get("N", 16),
                                     kw.get("K", 128), kw.get("G", 128), kw.get("P", A), A, A, None,
                                     kw.get("Y", A), kw.get("yd", 0), None, 0, None)
    assert g(M=0) == 1
    assert g(K=100) == 1
    assert g(G=48) == 2          # group not served
    assert g(G=32, K=96) == 2    # groups of 32 need K a multiple of 64
    assert g(xd=0) == 2          # fp32 activations are not served
    assert g(yd=1) == 2          # fp16 output not served
    assert g(X=None) == 1
    assert g(Y=A + 4) == 1
    assert g(P=A + 2) == 1
    assert b"aligned" in lib.w4_last_error()


class _Item(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("group", ctypes.c_int),
                ("x_dtype", ctypes.c_int), ("y_dtype", ctypes.c_int), ("packed", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p), ("awq_s", ctypes.c_void_p),
                ("x_offset", ctypes.c_size_t), ("y_offset", ctypes.c_size_t)]


def test_batch_host_entry_rejects_before_enqueueing(lib):
    """w4a16_gemm_host_batch_async checks every item on the host (no device call
    happens before these rejections) and names the bad item."""
    P = ctypes.c_void_p
    lib.w4a16_gemm_host_batch_async.argtypes = [ctypes.POINTER(_Item), ctypes.c_int, P, P, ctypes.c_size_t, P, P,
                                                ctypes.c_size_t, P, ctypes.c_size_t, P]
    lib.w4a16_gemm_host_batch_async.restype = ctypes.c_int
    lib.w4_last_error.restype = ctypes.c_char_p

    def item(**kw):
        it = _Item(kw.get("M", 1), kw.get("N", 256), kw.get("K", 1024), kw.get("G", 128), kw.get("xd", 2),
                   kw.get("yd", 0), kw.get("P", A), A, A, None, kw.get("xo", 0), kw.get("yo", 0))
        return it

    def call(items, xb=1 << 20, yb=1 << 20, X=A, Y=A):
        arr = (_Item * max(len(items), 1))(*items)
        return lib.w4a16_gemm_host_batch_async(arr if items else None, len(items), A, X, xb, A, Y, yb, None, 0, None)

    assert call([]) == 1
    assert call([item()], X=None) == 1
    assert call([item()], Y=A + 8) == 1                   # staging buffers must be 16-byte aligned
    assert call([item(), item(M=0)]) == 1
    assert b"item 1" in lib.w4_last_error()
    assert call([item(xd=0)]) == 2                         # fp32 activations are not served
    assert call([item(yd=1)]) == 2                         # fp16 output is not served
    assert call([item(G=48)]) == 2
    assert call([item(P=A + 2)]) == 1
    assert call([item(xo=8)]) == 1                         # offsets are 16-byte multiples
    assert call([item(), item(xo=2064)], xb=4096) == 1     # item 1's 2048 bytes of X end past 4096
    assert b"item 1" in lib.w4_last_error() and b"outside" in lib.w4_last_error()
    assert call([item(xo=4096)], xb=4096) == 1
    assert b"outside" in lib.w4_last_error()
    assert call([item(N=256, yo=1024)], yb=1024 + 1023) == 1  # one row of 256 fp32 outputs needs 1024 bytes
    assert b"outside" in lib.w4_last_error()


def test_workspace_size_plan(lib):
    _setup(lib)
    # decode of a 14336-deep layer splits K across CTAs -> needs partials + counters
    assert lib.w4a16_gemm_workspace_size(1, 4096, 14336) > 4096 * 4
    # invalid shapes need none
    assert lib.w4a16_gemm_workspace_size(0, 16, 128) == 0
    assert lib.w4a16_gemm_workspace_size(1, 16, 100) == 0


def test_outlier_default_count_is_top_tenth_percent(lib):
    """The default count of the dense + sparse split is the top 0.1 % of the
    weights (mhpq.cn practitioner's article, section 2.2): ceil(N K / 1000), at
    least 1; a host-only helper, so it runs without a GPU."""
    lib.w4_outliers_default_count.argtypes = [ctypes.c_int64, ctypes.c_int64]
    lib.w4_outliers_default_count.restype = ctypes.c_int64
    f = lib.w4_outliers_default_count
    assert f(4096, 4096) == 16778          # 16777216 / 1000 rounded up
    assert f(28672, 4096) == 117441        # Llama-3-8B gate_up
    assert f(1000, 1) == 1 and f(1001, 1) == 2 and f(1, 1) == 1
    assert f(0, 128) == 0 and f(4, -1) == 0
