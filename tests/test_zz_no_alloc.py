"""GPU check of w4a16_gemm_decode_static, the decode GEMM whose scratch is a
fixed array inside the library (no workspace argument, nothing allocated by
the call).  Each case runs it twice in a row through the C ABI and compares
both results with w4a16_gemm (caller-owned workspace) on the same weights,
within the GEMM tolerance |y - y_ref| <= 2e-3 * sum_k |x w^|.

The file name sorts last so that the suite also runs this after every other
GPU test in one process; it passes alone in a fresh process as well."""
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


@pytest.mark.parametrize("M,N,K,awq", [
    (1, 256, 256, False),
    (1, 4096, 14336, False),   # split-K over k-slices: partials and counters in the scratch
    (4, 4096, 14336, True),
    (3, 1000, 4096, False),
    (16, 4096, 14336, False),
    (64, 4096, 14336, False),  # tensor-core plan with fewer K splits so its partials fit the scratch
])
def test_static_scratch_matches_workspace_entry(w4, M, N, K, awq):
    tag = ("noalloc", M, N, K, awq)
    W = synthetic.weight(K, N, 0.02, 0.001, tag)
    s = synthetic.awq_scale(K, tag) if awq else None
    X = synthetic.activations(M, K, "bf16", tag).cuda()
    sd = None if s is None else s.cuda()
    packed, scales, zeros = w4.w4_quantize(W.cuda(), sd)
    Yref = w4.w4a16_gemm(X, packed, scales, zeros, sd)
    Y1 = w4.w4a16_gemm_decode_static(X, packed, scales, zeros, sd)
    Y2 = w4.w4a16_gemm_decode_static(X, packed, scales, zeros, sd)
    torch.cuda.synchronize()
    # sum_k |x w^| from the oracle's dequantized weights bounds the error
    codes, sc, zp = oracle.quantize(W.numpy(), None if s is None else s.numpy())
    What = oracle.dequant(codes, sc, zp, None if s is None else s.numpy())
    _, bound = oracle.gemm(X.float().cpu().numpy(), What)
    ref = Yref.cpu().numpy().astype(np.float64)
    for Y in (Y1, Y2):
        check_close(Y.cpu().numpy(), ref, bound, what=f"static scratch M={M} N={N} K={K}")
    assert w4.w4_device_error() == 0


def test_static_scratch_rejects_oversized_plan(w4):
    """M=8 on a wide, deep layer splits K into slices, and its fp32 partials
    (slices x 2 slots x 8 x 65536 floats) exceed the fixed scratch: rejected on
    the host with the sizes in the message (buffers are full-size all the same)."""
    M, N, K = 8, 65536, 8192
    assert w4.w4a16_gemm_workspace_size(M, N, K) > w4.w4a16_gemm_decode_static_capacity()
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((N, K // 128), dtype=torch.float16, device="cuda")
    with pytest.raises(w4.W4Error) as ei:
        w4.w4a16_gemm_decode_static(X, packed, sc, sc)
    assert ei.value.status == w4.W4_ERR_UNSUPPORTED
    assert "static scratch" in str(ei.value)
    del packed, sc
    torch.cuda.empty_cache()


def test_static_scratch_rejects_prefill_shapes(w4):
    X = torch.zeros((65, 256), dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros((128, 128), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((128, 2), dtype=torch.float16, device="cuda")
    with pytest.raises(w4.W4Error) as ei:
        w4.w4a16_gemm_decode_static(X, packed, sc, sc)
    assert ei.value.status == w4.W4_ERR_UNSUPPORTED
