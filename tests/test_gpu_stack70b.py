"""Whole-model 70B decode step (80 Llama-3-70B layers plus lm_head, 36.9 GB
packed) against the oracle. It runs at full size, in the launch configuration
the bench times.

The stack is quantized on the device one matrix at a time. Three rows of every
dense matrix are copied to the host before that, and for those rows:
  * packed codes, scales and zeros must equal the oracle's bit for bit;
  * the outputs of one decode step at M=1 and at M=16, taken after every
    linear layer, must be within |y - y_ref| <= 2e-3 * sum_k |x w^| of the
    oracle's matmul.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_int4_w4_b200 import stack70b

from ._util import check_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    from weight_only_int4_w4_b200 import w4 as mod
    return mod


@pytest.fixture(scope="module")
def stack(w4):
    layers, q_ms, q_bytes = stack70b.build(w4, keep=3)
    yield layers
    del layers
    torch.cuda.empty_cache()


def test_stack_shape(stack):
    assert len(stack) == 4 * 80 + 1
    params = sum(L["N"] * L["K"] for L in stack)
    assert params == 69_501_714_432
    packed_bytes = sum(L["packed"].numel() + 2 * L["scales"].numel() + 2 * L["zeros"].numel() for L in stack)
    assert abs(packed_bytes / 1e9 - 36.92) < 0.01


def test_stack_quantize_rows_bit_exact(stack):
    for L in stack:
        rows = torch.from_numpy(L["rows"]).cuda()
        codes, sc, zp = oracle.quantize(L["W_rows"].numpy())
        what = f"layer {L['i']} {L['name']}"
        assert np.array_equal(L["packed"][rows].cpu().numpy(), oracle.pack(codes)), f"{what}: packed"
        assert np.array_equal(L["scales"][rows].view(torch.int16).cpu().numpy().view(np.uint16),
                              sc.view(np.uint16)), f"{what}: scales"
        assert np.array_equal(L["zeros"][rows].view(torch.int16).cpu().numpy().view(np.uint16),
                              zp.view(np.uint16)), f"{what}: zeros"


@pytest.mark.parametrize("M", [1, 16])
def test_stack_decode_step(w4, stack, M):
    X, Y, ws = stack70b.step_buffers(w4, stack, M)
    got = []
    stack70b.run_step(w4, stack, X, Y, ws,
                      after_layer=lambda L, y: got.append(y[:, torch.from_numpy(L["rows"]).cuda()].clone()))
    torch.cuda.synchronize()
    assert w4.w4_device_error() == 0
    for L, g in zip(stack, got):
        codes, sc, zp = oracle.quantize(L["W_rows"].numpy())
        What = oracle.dequant(codes, sc, zp)
        Yref, bound = oracle.gemm(X[L["K"]].float().cpu().numpy(), What)
        check_close(g.cpu().numpy(), Yref, bound, what=f"M={M} layer {L['i']} {L['name']}")
