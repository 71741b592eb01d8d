"""GPU parity of the dense + sparse outlier split against the oracle.

The split keeps the top-|w| weights in fp16 CSR and quantizes the rest with
those weights taken as 0. The dense codes, scales, zeros and packed bytes and
the CSR must equal the oracle's exactly. The GEMM with the sparse part added
must hold |y - y_ref| <= 2e-3 * sum_k |x w^| per element, with W^ including
the fp16 outliers.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from weight_only_int4_w4_b200 import synthetic

from ._util import check_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    from weight_only_int4_w4_b200 import w4 as mod
    return mod


def _u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("N,K,awq,frac,group", [(256, 256, False, 0.001, 128), (4096, 4096, False, 0.001, 128),
                                                (300, 1024, True, 0.002, 128), (6144, 4096, False, 0.001, 128),
                                                (512, 1024, False, 0.002, 64), (256, 512, True, 0.002, 32)])
def test_outlier_split_bit_exact(w4, N, K, awq, frac, group):
    tag = ("outliers", N, K, awq, group)
    W = synthetic.weight(K, N, 0.02, 0.001, tag)
    s = synthetic.awq_scale(K, tag) if awq else None
    count = int(np.ceil(frac * N * K))
    packed, scales, zeros, (row_ptr, col, val) = w4.w4_quantize_outliers(
        W.cuda(), count, None if s is None else s.cuda(), group=group)
    torch.cuda.synchronize()
    c, sc, zp, rp, cl, vl = oracle.outlier_split(W.numpy(), count, None if s is None else s.numpy(), group=group)
    assert np.array_equal(row_ptr.cpu().numpy(), rp)
    assert np.array_equal(col.cpu().numpy(), cl)
    assert np.array_equal(_u16(val), vl.view(np.uint16))
    assert np.array_equal(packed.cpu().numpy(), oracle.pack(c))
    assert np.array_equal(_u16(scales), sc.view(np.uint16))
    assert np.array_equal(_u16(zeros), zp.view(np.uint16))


@pytest.mark.parametrize("M", [1, 5, 300])
def test_gemm_with_outliers(w4, M):
    N, K = 1024, 2048
    tag = ("outliers-gemm", M)
    W = synthetic.weight(K, N, 0.02, 0.002, tag)
    X = synthetic.activations(M, K, "bf16", tag)
    count = int(np.ceil(0.001 * N * K))
    packed, scales, zeros, csr = w4.w4_quantize_outliers(W.cuda(), count)
    Y = w4.w4a16_gemm_outliers(X.cuda(), packed, scales, zeros, csr)
    torch.cuda.synchronize()
    c, sc, zp, rp, cl, vl = oracle.outlier_split(W.numpy(), count)
    What = oracle.outlier_dequant(c, sc, zp, rp, cl, vl)
    Yref, bound = oracle.gemm(X.float().numpy(), What)
    check_close(Y.cpu().numpy(), Yref, bound, what=f"outliers M={M}")


def test_outlier_ties_and_capacity(w4):
    """Three equal largest magnitudes with count 2: all three are kept. A capacity of 2
    is reported as too small with the true entry count, and nothing is written past it."""
    W = torch.full((2, 128), 0.01)
    W[0, 3] = W[1, 7] = W[1, 9] = 0.5
    packed, scales, zeros, (row_ptr, col, val) = w4.w4_quantize_outliers(W.cuda(), 2)
    assert row_ptr.cpu().tolist() == [0, 1, 3] and col.cpu().tolist() == [3, 7, 9]
    Wd = W.cuda()
    cap = 2
    col2 = torch.full((cap + 4,), -1, dtype=torch.int32, device="cuda")
    val2 = torch.zeros(cap + 4, dtype=torch.float16, device="cuda")
    rp2 = torch.empty(3, dtype=torch.int32, device="cuda")
    ws = torch.zeros(int(w4.lib.w4_outliers_workspace_size(2)), dtype=torch.uint8, device="cuda")
    nnz = ctypes.c_int64(0)
    P = ctypes.c_void_p
    st = w4.lib.w4_quantize_outliers(P(Wd.data_ptr()), None, 2, 128, 128, 2, P(packed.data_ptr()),
                                     P(scales.data_ptr()), P(zeros.data_ptr()), P(rp2.data_ptr()), P(col2.data_ptr()),
                                     P(val2.data_ptr()), cap, ctypes.cast(ctypes.pointer(nnz), P), P(ws.data_ptr()),
                                     ws.numel(), P(torch.cuda.current_stream().cuda_stream))
    assert st == w4.W4_ERR_INVALID_ARG and nnz.value == 3
    assert col2.cpu().tolist()[cap:] == [-1] * 4


def test_no_device_error(w4):
    assert w4.w4_device_error() == 0
