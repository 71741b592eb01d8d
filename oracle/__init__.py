"""CPU oracle for weight-only per-group INT4 (W4A16): test infrastructure only.

Only the test-suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The product path (the CUDA library and
its Python binding) never imports it, and it imports nothing from the product.

The arithmetic lives in ``w4_oracle.c`` (plain C loops, fp32 quantize with
round-half-even, fp64 matmul accumulation); this module only compiles it with
gcc and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w4_oracle.c")
_LIB = os.path.join(_HERE, "libw4oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-frounding-math", _SRC, "-o", _LIB, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        _lib.w4o_quantize.argtypes = [P, P, I64, I64, ctypes.c_int, P, P, P]
        _lib.w4o_quantize_sym.argtypes = [P, P, I64, I64, ctypes.c_int, P, P, P]
        _lib.w4o_awq_search.argtypes = [P, I64, I64, ctypes.c_int, P, I64, P, ctypes.c_int, P, P, P]
        _lib.w4o_gptq.argtypes = [P, I64, I64, ctypes.c_int, P, I64, ctypes.c_double, P, P, P]
        _lib.w4o_pack.argtypes = [P, I64, I64, P]
        _lib.w4o_unpack.argtypes = [P, I64, I64, P]
        _lib.w4o_dequant.argtypes = [P, P, P, P, I64, I64, ctypes.c_int, P]
        _lib.w4o_gemm.argtypes = [P, P, I64, I64, I64, P, P]
        _lib.w4o_f32_to_f16.argtypes = [ctypes.c_float]
        _lib.w4o_f32_to_f16.restype = ctypes.c_uint16
        _lib.w4o_f16_to_f32.argtypes = [ctypes.c_uint16]
        _lib.w4o_f16_to_f32.restype = ctypes.c_float
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def quantize(W, awq_s=None, group: int = 128):
    """W [N,K] float32 (optionally AWQ s [K]) -> (codes u8 [N,K], scales f16 [N,K/G], zeros f16 [N,K/G])."""
    W = _c(W, np.float32)
    s = _c(awq_s, np.float32)
    N, K = W.shape
    codes = np.empty((N, K), np.uint8)
    scales = np.empty((N, K // group), np.uint16)
    zeros = np.empty((N, K // group), np.uint16)
    rc = _load().w4o_quantize(_ptr(W), _ptr(s), N, K, group, _ptr(codes), _ptr(scales), _ptr(zeros))
    if rc != 0:
        raise ValueError("w4o_quantize rejected its arguments")
    return codes, scales.view(np.float16), zeros.view(np.float16)


def quantize_symmetric(W, awq_s=None, group: int = 128):
    """Symmetric variant: codes q + 8 with q in [-7, 7], scale = fp16(max|w'| / 7), zeros all 8."""
    W = _c(W, np.float32)
    s = _c(awq_s, np.float32)
    N, K = W.shape
    codes = np.empty((N, K), np.uint8)
    scales = np.empty((N, K // group), np.uint16)
    zeros = np.empty((N, K // group), np.uint16)
    rc = _load().w4o_quantize_sym(_ptr(W), _ptr(s), N, K, group, _ptr(codes), _ptr(scales), _ptr(zeros))
    if rc != 0:
        raise ValueError("w4o_quantize_sym rejected its arguments")
    return codes, scales.view(np.float16), zeros.view(np.float16)


def awq_search(W, X, alphas, group: int = 128):
    """AWQ exponent search: W [N,K] fp32, X [Mc,K] (values of 16-bit inputs, as floats),
    alphas (exponent grid) -> (errors fp64 [n_alpha], s fp32 [K] of the best, best index)."""
    W = _c(W, np.float32)
    X = _c(X, np.float32)
    a = _c(np.asarray(alphas, np.float64), np.float64)
    N, K = W.shape
    Mc = X.shape[0]
    errors = np.empty(len(a), np.float64)
    s = np.empty(K, np.float32)
    best = ctypes.c_int(-1)
    rc = _load().w4o_awq_search(_ptr(W), N, K, group, _ptr(X), Mc, _ptr(a), len(a), _ptr(errors), _ptr(s),
                                ctypes.byref(best))
    if rc != 0:
        raise ValueError("w4o_awq_search rejected its arguments")
    return errors, s, best.value


def outlier_split(W, count, awq_s=None, group: int = 128):
    """Dense + sparse split (mhpq.cn article, section 2.2): every weight with |w| >= tau, tau the
    count-th largest |w| (ties all kept), goes to an fp16 sparse part; the rest is quantized with
    those weights taken as 0.  Plain numpy selection (full sort) and the C quantizer.
    Returns (codes, scales, zeros, row_ptr int32 [N+1], col int32 [nnz], val fp16 [nnz])."""
    W = _c(W, np.float32)
    N, K = W.shape
    mag = np.abs(W)
    tau = np.sort(mag, axis=None)[::-1][count - 1]
    mask = mag >= tau
    codes, scales, zeros = quantize(np.where(mask, np.float32(0.0), W), awq_s, group)
    rows, cols = np.nonzero(mask)  # row-major: increasing k within each row
    row_ptr = np.zeros(N + 1, np.int64)
    np.add.at(row_ptr, rows + 1, 1)
    row_ptr = np.cumsum(row_ptr).astype(np.int32)
    return codes, scales, zeros, row_ptr, cols.astype(np.int32), W[rows, cols].astype(np.float16)


def outlier_dequant(codes, scales, zeros, row_ptr, col, val, awq_s=None, group: int = 128):
    """W^ = dequant(dense) + sparse: the fp16 entries added at their positions."""
    What = dequant(codes, scales, zeros, awq_s, group)
    N = What.shape[0]
    rows = np.repeat(np.arange(N), np.diff(row_ptr.astype(np.int64)))
    What[rows, col] += val.astype(np.float32)
    return What


def gptq(W, X, group: int = 128, damp_frac: float = 0.01):
    """GPTQ column sweep with Hessian 2 X^T X (plain fp64 loops): W [N,K] fp32, X [Mc,K] floats
    -> (codes u8 [N,K], scales f16 [N,K/G], zeros f16 [N,K/G])."""
    W = _c(W, np.float32)
    X = _c(X, np.float32)
    N, K = W.shape
    codes = np.empty((N, K), np.uint8)
    scales = np.empty((N, K // group), np.uint16)
    zeros = np.empty((N, K // group), np.uint16)
    rc = _load().w4o_gptq(_ptr(W), N, K, group, _ptr(X), X.shape[0], float(damp_frac), _ptr(codes), _ptr(scales),
                          _ptr(zeros))
    if rc != 0:
        raise ValueError(f"w4o_gptq failed ({rc})")
    return codes, scales.view(np.float16), zeros.view(np.float16)


def pack(codes):
    codes = _c(codes, np.uint8)
    N, K = codes.shape
    packed = np.empty((N, K // 2), np.uint8)
    if _load().w4o_pack(_ptr(codes), N, K, _ptr(packed)) != 0:
        raise ValueError("w4o_pack rejected its arguments")
    return packed


def unpack(packed, K: int):
    packed = _c(packed, np.uint8)
    N = packed.shape[0]
    codes = np.empty((N, K), np.uint8)
    if _load().w4o_unpack(_ptr(packed), N, K, _ptr(codes)) != 0:
        raise ValueError("w4o_unpack rejected its arguments")
    return codes


def dequant(codes, scales, zeros, awq_s=None, group: int = 128):
    codes = _c(codes, np.uint8)
    sc = _c(np.asarray(scales, np.float16).view(np.uint16), np.uint16)
    zp = _c(np.asarray(zeros, np.float16).view(np.uint16), np.uint16)
    s = _c(awq_s, np.float32)
    N, K = codes.shape
    What = np.empty((N, K), np.float32)
    if _load().w4o_dequant(_ptr(codes), _ptr(sc), _ptr(zp), _ptr(s), N, K, group, _ptr(What)) != 0:
        raise ValueError("w4o_dequant rejected its arguments")
    return What


def gemm(X, What):
    """X [M,K] (values of fp16/bf16 inputs, widened), W^ [N,K] -> (Y fp64 [M,N], bound fp64 [M,N])."""
    X = _c(X, np.float32)
    What = _c(What, np.float32)
    M, K = X.shape
    N = What.shape[0]
    Y = np.empty((M, N), np.float64)
    B = np.empty((M, N), np.float64)
    if _load().w4o_gemm(_ptr(X), _ptr(What), M, N, K, _ptr(Y), _ptr(B)) != 0:
        raise ValueError("w4o_gemm rejected its arguments")
    return Y, B


def f32_to_f16_bits(v: float) -> int:
    return int(_load().w4o_f32_to_f16(float(v)))


def f16_bits_to_f32(b: int) -> float:
    return float(_load().w4o_f16_to_f32(int(b)))


def reference_linear(X, W, awq_s=None, group: int = 128):
    """Whole path on the CPU: quantize W, dequantize, and Y = X . W^T (fp64)."""
    codes, scales, zeros = quantize(W, awq_s, group)
    What = dequant(codes, scales, zeros, awq_s, group)
    Y, bound = gemm(X, What)
    return Y, bound, (codes, scales, zeros, What)
