"""GPU parity of the quantizer variants against the oracle.

Two variants are covered. The symmetric one stores INT4 as {-7..7} + 8 with
zero point 8. The asymmetric and symmetric quantizers are also run with groups
of 32 and 64 channels. Codes, scales, zeros and packed bytes must equal the
oracle's bit for bit. The GEMM on these weights must hold
|y - y_ref| <= 2e-3 * sum_k |x w^| per element.
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
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _quant_both(w4, W, s, group, symmetric):
    packed, scales, zeros, codes = w4.w4_quantize(W.cuda(), None if s is None else s.cuda(), group=group,
                                                  return_codes=True, symmetric=symmetric)
    torch.cuda.synchronize()
    fn = oracle.quantize_symmetric if symmetric else oracle.quantize
    c, sc, zp = fn(W.numpy(), None if s is None else s.numpy(), group=group)
    return (packed, scales, zeros, codes), (c, sc, zp)


@pytest.mark.parametrize("symmetric", [False, True])
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("N,K,awq", [(256, 256, False), (300, 1024, True), (6144, 4096, False), (7, 96, False)])
def test_quantize_variants_bit_exact(w4, symmetric, group, N, K, awq):
    if K % group:
        pytest.skip("K not a multiple of the group")
    tag = ("variants", N, K, group, symmetric)
    W = synthetic.weight(K, N, 0.02, 0.001, tag)
    s = synthetic.awq_scale(K, tag) if awq else None
    (packed, scales, zeros, codes), (c, sc, zp) = _quant_both(w4, W, s, group, symmetric)
    what = f"N={N} K={K} G={group} sym={symmetric} awq={awq}"
    assert np.array_equal(codes.cpu().numpy(), c), f"{what}: codes"
    assert np.array_equal(_u16(scales), sc.view(np.uint16)), f"{what}: scales"
    assert np.array_equal(_u16(zeros), zp.view(np.uint16)), f"{what}: zeros"
    assert np.array_equal(packed.cpu().numpy(), oracle.pack(c)), f"{what}: packed"


def test_symmetric_codes_range_and_zero(w4):
    W = synthetic.weight(1024, 512, 0.02, 0.001, ("symrange",))
    packed, scales, zeros, codes = w4.w4_quantize(W.cuda(), return_codes=True, symmetric=True)
    c = codes.cpu().numpy()
    assert c.min() >= 1 and c.max() <= 15
    assert torch.all(zeros.float() == 8.0)


@pytest.mark.parametrize("symmetric", [False, True])
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("M,N,K", [(1, 384, 1024), (5, 300, 512), (64, 256, 768), (300, 200, 1280)])
def test_gemm_on_variant_weights(w4, symmetric, group, M, N, K):
    tag = ("variants-gemm", M, N, K, group, symmetric)
    W = synthetic.weight(K, N, 0.02, 0.0, tag)
    X = synthetic.activations(M, K, "bf16", tag)
    packed, scales, zeros = w4.w4_quantize(W.cuda(), group=group, symmetric=symmetric)
    Y = w4.w4a16_gemm(X.cuda(), packed, scales, zeros, group=group)
    torch.cuda.synchronize()
    fn = oracle.quantize_symmetric if symmetric else oracle.quantize
    c, sc, zp = fn(W.numpy(), group=group)
    What = oracle.dequant(c, sc, zp, group=group)
    Yref, bound = oracle.gemm(X.float().numpy(), What)
    check_close(Y.cpu().numpy(), Yref, bound, what=f"M={M} N={N} K={K} G={group} sym={symmetric}")


def test_group32_needs_k_multiple_of_64(w4):
    X = torch.zeros((1, 96), dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros((64, 48), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((64, 3), dtype=torch.float16, device="cuda")
    with pytest.raises(w4.W4Error) as ei:
        w4.w4a16_gemm(X, packed, sc, sc, group=32)
    assert ei.value.status == w4.W4_ERR_UNSUPPORTED


def test_no_device_error(w4):
    assert w4.w4_device_error() == 0


@pytest.mark.parametrize("group", [32, 64])
def test_tail_split_with_small_groups(w4, monkeypatch, capfd, group):
    """The tensor-core tail split (the last, mostly empty wave's tiles cut into
    k-pieces summed by a reduction kernel) with groups of 32 and 64: every
    output of the tail tiles, plus sampled rows elsewhere, against the oracle."""
    monkeypatch.setenv("W4_DEBUG_PLAN", "1")
    M, N, K = 300, 9688, 2048
    tag = ("variants-tail", group)
    W = synthetic.weight(K, N, 0.02, 0.0, tag)
    X = synthetic.activations(M, K, "bf16", tag)
    packed, scales, zeros = w4.w4_quantize(W.cuda(), group=group)
    Y = w4.w4a16_gemm(X.cuda(), packed, scales, zeros, group=group)
    torch.cuda.synchronize()
    ntx = (N + 127) // 128
    tiles = ntx * 2  # BN = 256 for M = 300
    head = tiles - tiles % 148
    tail_rows = {n for t in range(head, tiles) for n in range((t % ntx) * 128, min((t % ntx) * 128 + 128, N))}
    rows = np.array(sorted(tail_rows | set(np.random.default_rng(group).choice(N, 48, replace=False).tolist())))
    c, sc, zp = oracle.quantize(W.numpy()[rows], group=group)
    What = oracle.dequant(c, sc, zp, group=group)
    Yref, bound = oracle.gemm(X.float().numpy(), What)
    check_close(Y.cpu().numpy()[:, rows], Yref, bound, what=f"tail G={group}")
    err = capfd.readouterr().err
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert f"head_tiles={head} tail_pieces=2 " in err, err
