"""GPU parity of the GPTQ column sweep (w4_quantize_gptq) against the oracle's
plain fp64 loops.

Both sides evaluate the same operations in the same order, without fused
multiply-adds: the Hessian, the damping, the Cholesky factor of the reversed
Hessian, its triangular inverse, and the per-row sweep with fp32 code
decisions. The codes, scales, zeros and packed bytes must therefore be equal
bit for bit. The GEMM on GPTQ weights holds the usual element-wise bound.
"""
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


def _calibration(Mc, K, tag):
    """bf16 N(0,1) activations with correlated channels (a non-diagonal Hessian)."""
    g = torch.Generator().manual_seed(synthetic.seed_of(tag, "gptq-calib") % (2 ** 62))
    X = torch.randn((Mc, K), generator=g)
    X += 0.5 * X[:, :1]
    return X.to(torch.bfloat16)


@pytest.mark.parametrize("N,K,Mc,group", [(64, 256, 128, 128), (40, 512, 96, 64), (33, 128, 64, 32),
                                          (200, 1024, 128, 128)])
def test_gptq_bit_exact(w4, N, K, Mc, group):
    tag = ("gptq", N, K, Mc, group)
    W = synthetic.weight(K, N, 0.02, 0.001, tag)
    X = _calibration(Mc, K, tag)
    packed, scales, zeros, codes = w4.w4_quantize_gptq(W.cuda(), X.cuda(), group=group, return_codes=True)
    torch.cuda.synchronize()
    c, sc, zp = oracle.gptq(W.numpy(), X.float().numpy(), group=group)
    assert np.array_equal(codes.cpu().numpy(), c)
    assert np.array_equal(_u16(scales), sc.view(np.uint16))
    assert np.array_equal(_u16(zeros), zp.view(np.uint16))
    assert np.array_equal(packed.cpu().numpy(), oracle.pack(c))


def test_gptq_weights_through_the_gemm_and_objective(w4):
    """The GEMM consumes GPTQ weights like any others. The layer-output error on
    the calibration batch is below plain RTN's."""
    N, K, Mc = 256, 512, 128
    tag = ("gptq-gemm",)
    W = synthetic.weight(K, N, 0.02, 0.0, tag)
    X = _calibration(Mc, K, tag)
    packed, scales, zeros, codes = w4.w4_quantize_gptq(W.cuda(), X.cuda(), return_codes=True)
    Y = w4.w4a16_gemm(X.cuda(), packed, scales, zeros)
    torch.cuda.synchronize()
    c, sc, zp = oracle.gptq(W.numpy(), X.float().numpy())
    What = oracle.dequant(c, sc, zp)
    Yref, bound = oracle.gemm(X.float().numpy(), What)
    check_close(Y.cpu().numpy(), Yref, bound, what="gptq gemm")
    Yexact, _ = oracle.gemm(X.float().numpy(), W.numpy())
    cr, sr, zr = oracle.quantize(W.numpy())
    Yrtn, _ = oracle.gemm(X.float().numpy(), oracle.dequant(cr, sr, zr))
    assert np.sum((Yexact - Yref) ** 2) < 0.7 * np.sum((Yexact - Yrtn) ** 2)


def test_gptq_rejects_a_singular_hessian(w4):
    """All-zero calibration: H = 0 and the damping (a fraction of its trace) is 0."""
    W = torch.randn((16, 128), device="cuda") * 0.02
    X = torch.zeros((8, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w4.W4Error) as ei:
        w4.w4_quantize_gptq(W, X)
    assert ei.value.status == w4.W4_ERR_INVALID_ARG
    assert "positive definite" in str(ei.value)


def test_no_device_error(w4):
    assert w4.w4_device_error() == 0
