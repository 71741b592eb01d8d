"""Python binding of libw4 (argument marshalling only).

Every function here forwards torch tensors' device pointers, sizes and the
current CUDA stream to the C ABI declared in ``include/w4.h``; all arithmetic
runs in the library's CUDA kernels.  There is no fallback: if ``libw4.so`` is
not built, importing this module raises.

Names follow the C ABI: ``w4_quantize`` (and ``w4_quantize_symmetric``), ``w4_pack``, ``w4a16_gemm``,
``w4a16_gemm_workspace_size``, ``w4a16_gemm_host``, ``w4a16_gemm_decode_static``,
``w4_device_error``.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libw4.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libw4.so is not built ({_LIB_PATH}); run weight_only_int4_w4_b200.build.build_library()")

_lib = ctypes.CDLL(_LIB_PATH)
_P, _I64, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
_lib.w4_quantize.argtypes = [_P, ctypes.c_int, _P, _I64, _I64, ctypes.c_int, _P, _P, _P, _P, _P]
_lib.w4_quantize_symmetric.argtypes = [_P, ctypes.c_int, _P, _I64, _I64, ctypes.c_int, _P, _P, _P, _P, _P]
_lib.w4_pack.argtypes = [_P, _I64, _I64, _P, _P]
_lib.w4a16_gemm.argtypes = [_P, ctypes.c_int, _I64, _I64, _I64, ctypes.c_int, _P, _P, _P, _P, _P, ctypes.c_int,
                            _P, _SZ, _P]
_lib.w4a16_gemm_host.argtypes = [_P, _P, ctypes.c_int, _I64, _I64, _I64, ctypes.c_int, _P, _P, _P, _P, _P, _P,
                                 ctypes.c_int, _P, _SZ, _P]
_lib.w4a16_gemm_host_async.argtypes = _lib.w4a16_gemm_host.argtypes
_lib.w4a16_gemm_decode_static.argtypes = [_P, ctypes.c_int, _I64, _I64, _I64, ctypes.c_int, _P, _P, _P, _P, _P,
                                          ctypes.c_int, _P]
_lib.w4a16_gemm_decode_static_capacity.argtypes = []
_lib.w4a16_gemm_decode_static_capacity.restype = _SZ
_lib.w4_awq_search.argtypes = [_P, _I64, _I64, ctypes.c_int, _P, ctypes.c_int, _I64, _P, ctypes.c_int, _P, _P, _P,
                               _P, _SZ, _P]
_lib.w4_awq_search_workspace_size.argtypes = [_I64, _I64, _I64, ctypes.c_int]
_lib.w4_awq_search_workspace_size.restype = _SZ
_lib.w4_quantize_outliers.argtypes = [_P, _P, _I64, _I64, ctypes.c_int, _I64, _P, _P, _P, _P, _P, _P, _I64, _P, _P,
                                      _SZ, _P]
_lib.w4_outliers_workspace_size.argtypes = [_I64]
_lib.w4_outliers_workspace_size.restype = _SZ
_lib.w4_outliers_default_count.argtypes = [_I64, _I64]
_lib.w4_outliers_default_count.restype = _I64
_lib.w4a16_gemm_outliers.argtypes = [_P, ctypes.c_int, _I64, _I64, _I64, ctypes.c_int, _P, _P, _P, _P, _P, _P, _P,
                                     _P, ctypes.c_int, _P, _SZ, _P]
_lib.w4_quantize_gptq.argtypes = [_P, _I64, _I64, ctypes.c_int, _P, ctypes.c_int, _I64, ctypes.c_double, _P, _P, _P,
                                  _P, _P, _SZ, _P]
_lib.w4_gptq_workspace_size.argtypes = [_I64, _I64]
_lib.w4_gptq_workspace_size.restype = _SZ
_lib.w4a16_gemm_workspace_size.argtypes = [_I64, _I64, _I64]
_lib.w4a16_gemm_workspace_size.restype = _SZ


class GemmItem(ctypes.Structure):
    """w4_gemm_item of include/w4.h: one matmul of a host-buffer batch."""
    _fields_ = [("M", _I64), ("N", _I64), ("K", _I64), ("group", ctypes.c_int), ("x_dtype", ctypes.c_int),
                ("y_dtype", ctypes.c_int), ("packed", _P), ("scales", _P), ("zeros", _P), ("awq_s", _P),
                ("x_offset", _SZ), ("y_offset", _SZ)]


_lib.w4a16_gemm_host_batch_async.argtypes = [ctypes.POINTER(GemmItem), ctypes.c_int, _P, _P, _SZ, _P, _P, _SZ, _P,
                                             _SZ, _P]
_lib.w4_device_error.argtypes = [ctypes.POINTER(ctypes.c_int)]
_lib.w4_status_string.argtypes = [ctypes.c_int]
_lib.w4_status_string.restype = ctypes.c_char_p
_lib.w4_last_error.restype = ctypes.c_char_p
for _f in ("w4_quantize", "w4_quantize_symmetric", "w4_awq_search", "w4_quantize_outliers", "w4a16_gemm_outliers",
           "w4_quantize_gptq",
           "w4_pack", "w4a16_gemm", "w4a16_gemm_host", "w4a16_gemm_host_async", "w4a16_gemm_host_batch_async",
           "w4a16_gemm_decode_static", "w4_device_error"):
    getattr(_lib, _f).restype = ctypes.c_int

W4_OK, W4_ERR_INVALID_ARG, W4_ERR_UNSUPPORTED, W4_ERR_CUDA = 0, 1, 2, 3
W4_F32, W4_F16, W4_BF16 = 0, 1, 2
_DT = {torch.float32: W4_F32, torch.float16: W4_F16, torch.bfloat16: W4_BF16}
GROUP = 128

LIB_PATH = _LIB_PATH
lib = _lib


class W4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.w4_last_error().decode()
        super().__init__(f"{where}: {_lib.w4_status_string(status).decode()}: {msg}")


def _check(status: int, where: str):
    if status != W4_OK:
        raise W4Error(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def w4_status_string(status: int) -> str:
    return _lib.w4_status_string(status).decode()


def w4_quantize(W: torch.Tensor, awq_s: torch.Tensor | None = None, group: int = GROUP,
                return_codes: bool = False, stream=None, symmetric: bool = False, out=None):
    """Quantize + pack W [N, K] (fp32/fp16/bf16, CUDA).  Returns (packed u8 [N,K/2],
    scales f16 [N,K/G], zeros f16 [N,K/G]) and, with return_codes, codes u8 [N,K].
    symmetric=True calls w4_quantize_symmetric (codes q + 8, q in [-7, 7]).
    out = (packed, scales, zeros) writes into caller-owned tensors of those shapes."""
    assert W.is_cuda and W.dim() == 2 and W.is_contiguous() and W.dtype in _DT
    N, K = W.shape
    dev = W.device
    if out is not None:
        packed, scales, zeros = out
        assert packed.shape == (N, K // 2) and scales.shape == (N, K // group) and zeros.shape == (N, K // group)
    else:
        packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((N, K // group), dtype=torch.float16, device=dev)
        zeros = torch.empty((N, K // group), dtype=torch.float16, device=dev)
    codes = torch.empty((N, K), dtype=torch.uint8, device=dev) if return_codes else None
    if awq_s is not None:
        assert awq_s.is_cuda and awq_s.dtype == torch.float32 and awq_s.is_contiguous()
    fn, name = (_lib.w4_quantize_symmetric, "w4_quantize_symmetric") if symmetric else (_lib.w4_quantize, "w4_quantize")
    _check(fn(_ptr(W), _DT[W.dtype], _ptr(awq_s), N, K, group, _ptr(packed), _ptr(scales), _ptr(zeros), _ptr(codes),
              _stream(stream)), name)
    return (packed, scales, zeros, codes) if return_codes else (packed, scales, zeros)


def w4_pack(codes: torch.Tensor, stream=None) -> torch.Tensor:
    assert codes.is_cuda and codes.dtype == torch.uint8 and codes.dim() == 2 and codes.is_contiguous()
    N, K = codes.shape
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=codes.device)
    _check(_lib.w4_pack(_ptr(codes), N, K, _ptr(packed), _stream(stream)), "w4_pack")
    return packed


def w4a16_gemm_workspace_size(M: int, N: int, K: int) -> int:
    return int(_lib.w4a16_gemm_workspace_size(M, N, K))


_ws_lock = threading.Lock()
_ws_cache: dict = {}


def workspace(M: int, N: int, K: int, device, stream=None) -> torch.Tensor | None:
    """A workspace (cached per device and stream) large enough for (M, N, K), zero-filled
    when allocated.  Every call leaves its counters zero again, so it can be reused."""
    need = w4a16_gemm_workspace_size(M, N, K)
    if need == 0:
        return None
    s = stream if stream is not None else torch.cuda.current_stream(device)
    key = (torch.device(device), s.cuda_stream)
    with _ws_lock:
        buf = _ws_cache.get(key)
        if buf is None or buf.numel() < need:
            buf = torch.zeros(max(need, 1 << 20), dtype=torch.uint8, device=device)
            _ws_cache[key] = buf
    return buf


def w4a16_gemm(X: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
               awq_s: torch.Tensor | None = None, out_dtype=torch.float32, out: torch.Tensor | None = None,
               ws: torch.Tensor | None = None, group: int = GROUP, stream=None) -> torch.Tensor:
    """Y = X . W^T with W^ dequantized on the fly.  X [M,K] fp16/bf16 (CUDA)."""
    assert X.is_cuda and X.dim() == 2 and X.is_contiguous() and X.dtype in (torch.float16, torch.bfloat16)
    M, K = X.shape
    N = packed.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=X.device)
    if ws is None:
        ws = workspace(M, N, K, X.device, stream)
    _check(_lib.w4a16_gemm(_ptr(X), _DT[X.dtype], M, N, K, group, _ptr(packed), _ptr(scales), _ptr(zeros),
                           _ptr(awq_s), _ptr(out), _DT[out.dtype], _ptr(ws), 0 if ws is None else ws.numel(),
                           _stream(stream)), "w4a16_gemm")
    return out


def w4a16_gemm_host(X_host: torch.Tensor, X_dev: torch.Tensor, packed, scales, zeros, Y_host: torch.Tensor,
                    Y_dev: torch.Tensor, awq_s=None, ws=None, group: int = GROUP, stream=None,
                    wait: bool = True) -> torch.Tensor:
    """End-to-end call with pinned host X and Y: H2D copy, fused GEMM, D2H copy, and
    (wait=True) a wait for the stream.  With wait=False the work is only enqueued
    (w4a16_gemm_host_async): Y_host is valid after the caller synchronizes the stream."""
    M, K = X_host.shape
    N = packed.shape[0]
    if ws is None:
        ws = workspace(M, N, K, X_dev.device, stream)
    fn = _lib.w4a16_gemm_host if wait else _lib.w4a16_gemm_host_async
    _check(fn(_ptr(X_host), _ptr(X_dev), _DT[X_host.dtype], M, N, K, group, _ptr(packed), _ptr(scales), _ptr(zeros),
              _ptr(awq_s), _ptr(Y_host), _ptr(Y_dev), _DT[Y_host.dtype], _ptr(ws), 0 if ws is None else ws.numel(),
              _stream(stream)), "w4a16_gemm_host" if wait else "w4a16_gemm_host_async")
    return Y_host


def gemm_batch(items) -> ctypes.Array:
    """The w4_gemm_item array for w4a16_gemm_host_batch: one entry per matmul, each a dict
    with M, N, K, packed, scales, zeros, x_offset and y_offset (bytes into the staging
    buffers), and optionally awq_s, group (128), x_dtype (torch.bfloat16) and y_dtype
    (torch.float32).  Build it once and reuse it while the weights stay in place."""
    arr = (GemmItem * len(items))()
    for a, it in zip(arr, items):
        a.M, a.N, a.K = it["M"], it["N"], it["K"]
        a.group = it.get("group", GROUP)
        a.x_dtype = _DT[it.get("x_dtype", torch.bfloat16)]
        a.y_dtype = _DT[it.get("y_dtype", torch.float32)]
        a.packed, a.scales, a.zeros = it["packed"].data_ptr(), it["scales"].data_ptr(), it["zeros"].data_ptr()
        a.awq_s = it["awq_s"].data_ptr() if it.get("awq_s") is not None else None
        a.x_offset, a.y_offset = it["x_offset"], it["y_offset"]
    return arr


def w4a16_gemm_host_batch(batch: ctypes.Array, X_host: torch.Tensor, X_dev: torch.Tensor, Y_host: torch.Tensor,
                          Y_dev: torch.Tensor, ws=None, stream=None, wait: bool = True):
    """Independent matmuls with pinned host activations and outputs in one call
    (w4a16_gemm_host_batch_async): one copy of X_host into X_dev, the matmuls of `batch`
    (from gemm_batch) in order, one copy of Y_dev into Y_host.  The staging buffers are
    byte views (any dtype); with wait=False Y_host is valid after the caller
    synchronizes the stream."""
    xb, yb = X_host.numel() * X_host.element_size(), Y_host.numel() * Y_host.element_size()
    assert X_dev.numel() * X_dev.element_size() >= xb and Y_dev.numel() * Y_dev.element_size() >= yb
    _check(_lib.w4a16_gemm_host_batch_async(batch, len(batch), _ptr(X_host), _ptr(X_dev), xb, _ptr(Y_host),
                                            _ptr(Y_dev), yb, _ptr(ws), 0 if ws is None else ws.numel(),
                                            _stream(stream)), "w4a16_gemm_host_batch_async")
    if wait:
        (stream if stream is not None else torch.cuda.current_stream()).synchronize()
    return Y_host


def w4a16_gemm_decode_static(X: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                             awq_s: torch.Tensor | None = None, out_dtype=torch.float32,
                             out: torch.Tensor | None = None, group: int = GROUP, stream=None) -> torch.Tensor:
    """Decode-shape Y = X . W^T using the library's own fixed scratch (no workspace
    argument).  Calls on one device must not overlap in time."""
    assert X.is_cuda and X.dim() == 2 and X.is_contiguous() and X.dtype in (torch.float16, torch.bfloat16)
    M, K = X.shape
    N = packed.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=X.device)
    _check(_lib.w4a16_gemm_decode_static(_ptr(X), _DT[X.dtype], M, N, K, group, _ptr(packed), _ptr(scales),
                                         _ptr(zeros), _ptr(awq_s), _ptr(out), _DT[out.dtype], _stream(stream)),
           "w4a16_gemm_decode_static")
    return out


def w4a16_gemm_decode_static_capacity() -> int:
    return int(_lib.w4a16_gemm_decode_static_capacity())


def w4_quantize_outliers(W: torch.Tensor, count: int | None = None, awq_s: torch.Tensor | None = None,
                         group: int = GROUP, stream=None):
    """Dense + sparse split of W [N,K] fp32 (CUDA): the `count` largest |w| in fp16 CSR (None: the
    library's default, w4_outliers_default_count), the rest quantized.
    Returns (packed, scales, zeros, (row_ptr, col, val))."""
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous()
    N, K = W.shape
    dev = W.device
    cap = int(_lib.w4_outliers_default_count(N, K)) if count is None else int(count)
    count = 0 if count is None else int(count)
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((N, K // group), dtype=torch.float16, device=dev)
    zeros = torch.empty((N, K // group), dtype=torch.float16, device=dev)
    row_ptr = torch.empty(N + 1, dtype=torch.int32, device=dev)
    ws = torch.zeros(int(_lib.w4_outliers_workspace_size(N)), dtype=torch.uint8, device=dev)
    cap += 1024
    while True:
        col = torch.empty(cap, dtype=torch.int32, device=dev)
        val = torch.empty(cap, dtype=torch.float16, device=dev)
        nnz = ctypes.c_int64(0)
        st = _lib.w4_quantize_outliers(_ptr(W), _ptr(awq_s), N, K, group, count, _ptr(packed), _ptr(scales),
                                       _ptr(zeros), _ptr(row_ptr), _ptr(col), _ptr(val), cap,
                                       ctypes.cast(ctypes.pointer(nnz), _P), _ptr(ws), ws.numel(), _stream(stream))
        if st == W4_ERR_INVALID_ARG and nnz.value > cap:
            cap = nnz.value
            continue
        _check(st, "w4_quantize_outliers")
        break
    return packed, scales, zeros, (row_ptr, col[: nnz.value], val[: nnz.value])


def w4a16_gemm_outliers(X: torch.Tensor, packed, scales, zeros, csr, awq_s=None, out_dtype=torch.float32,
                        out: torch.Tensor | None = None, ws: torch.Tensor | None = None, group: int = GROUP,
                        stream=None) -> torch.Tensor:
    """Y = X . (dequant(dense) + sparse)^T with the CSR from w4_quantize_outliers."""
    assert X.is_cuda and X.dim() == 2 and X.is_contiguous() and X.dtype in (torch.float16, torch.bfloat16)
    M, K = X.shape
    N = packed.shape[0]
    row_ptr, col, val = csr
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=X.device)
    if ws is None:
        ws = workspace(M, N, K, X.device, stream)
    _check(_lib.w4a16_gemm_outliers(_ptr(X), _DT[X.dtype], M, N, K, group, _ptr(packed), _ptr(scales), _ptr(zeros),
                                    _ptr(awq_s), _ptr(row_ptr), _ptr(col), _ptr(val), _ptr(out), _DT[out.dtype],
                                    _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)), "w4a16_gemm_outliers")
    return out


def w4_quantize_gptq(W: torch.Tensor, Xcal: torch.Tensor, group: int = GROUP, damp_frac: float = 0.01,
                     return_codes: bool = False, stream=None):
    """GPTQ column sweep of W [N,K] fp32 with calibration Xcal [Mc,K] f16/bf16 (CUDA).
    Returns (packed, scales, zeros) and, with return_codes, codes u8 [N,K]."""
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous()
    assert Xcal.is_cuda and Xcal.dtype in (torch.float16, torch.bfloat16) and Xcal.is_contiguous()
    N, K = W.shape
    dev = W.device
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((N, K // group), dtype=torch.float16, device=dev)
    zeros = torch.empty((N, K // group), dtype=torch.float16, device=dev)
    codes = torch.empty((N, K), dtype=torch.uint8, device=dev) if return_codes else None
    ws = torch.empty(int(_lib.w4_gptq_workspace_size(N, K)), dtype=torch.uint8, device=dev)
    _check(_lib.w4_quantize_gptq(_ptr(W), N, K, group, _ptr(Xcal), _DT[Xcal.dtype], Xcal.shape[0], float(damp_frac),
                                 _ptr(packed), _ptr(scales), _ptr(zeros), _ptr(codes), _ptr(ws), ws.numel(),
                                 _stream(stream)), "w4_quantize_gptq")
    return (packed, scales, zeros, codes) if return_codes else (packed, scales, zeros)


AWQ_EXPONENTS = tuple(round(-1.0 + 0.1 * i, 1) for i in range(21))  # -1.0, -0.9, ..., 1.0


def w4_awq_search(W: torch.Tensor, Xcal: torch.Tensor, alphas=AWQ_EXPONENTS, group: int = GROUP, stream=None):
    """AWQ exponent search on calibration activations.  W [N,K] fp32, Xcal [Mc,K] f16/bf16 (CUDA).
    Returns (awq_s fp32 [K] on the device, best exponent, errors list)."""
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous()
    assert Xcal.is_cuda and Xcal.dtype in (torch.float16, torch.bfloat16) and Xcal.is_contiguous()
    N, K = W.shape
    Mc = Xcal.shape[0]
    a = (ctypes.c_float * len(alphas))(*alphas)
    errs = (ctypes.c_double * len(alphas))()
    best = ctypes.c_int(-1)
    s = torch.empty(K, dtype=torch.float32, device=W.device)
    ws = torch.zeros(int(_lib.w4_awq_search_workspace_size(Mc, N, K, group)), dtype=torch.uint8, device=W.device)
    _check(_lib.w4_awq_search(_ptr(W), N, K, group, _ptr(Xcal), _DT[Xcal.dtype], Mc, ctypes.cast(a, _P), len(alphas),
                              _ptr(s), ctypes.cast(errs, _P), ctypes.cast(ctypes.pointer(best), _P), _ptr(ws),
                              ws.numel(), _stream(stream)), "w4_awq_search")
    return s, alphas[best.value], list(errs)


def w4_device_error() -> int:
    flag = ctypes.c_int(0)
    _check(_lib.w4_device_error(ctypes.byref(flag)), "w4_device_error")
    return flag.value
