"""GPU parity of K0 (quantize + pack) and of w4_pack: bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from weight_only_int4_w4_b200 import synthetic

from ._util import G, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    from weight_only_int4_w4_b200 import w4 as mod
    return mod


def _gpu_quant(w4, W, awq=None, dtype=torch.float32):
    Wd = W.to(dtype).cuda()
    sd = None if awq is None else awq.cuda()
    packed, scales, zeros, codes = w4.w4_quantize(Wd, sd, return_codes=True)
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (packed, scales.view(torch.uint16), zeros.view(torch.uint16), codes)]


def _assert_exact(gpu, W_np, awq_np=None, what=""):
    packed, scales, zeros, codes = gpu
    c, s, z = oracle.quantize(W_np, awq_np)
    assert np.array_equal(codes, c), f"{what}: codes differ at {np.argwhere(codes != c)[:5]}"
    assert np.array_equal(scales, s.view(np.uint16)), f"{what}: scales differ"
    assert np.array_equal(zeros, z.view(np.uint16)), f"{what}: zeros differ"
    assert np.array_equal(packed, oracle.pack(c)), f"{what}: packed bytes differ"


def test_tiny_workload_exact(w4):
    W = synthetic.weight(256, 256, 0.02, 0.0, ("tiny", "tiny"))
    _assert_exact(_gpu_quant(w4, W), W.numpy(), what="tiny")


@pytest.mark.parametrize("layer", list(synthetic.SHAPES_8B))
def test_decode_8b_layers_exact_full(w4, layer):
    """Every code, scale, zero and byte of the 8B-shaped layers (0.1% outliers)."""
    K, N = synthetic.SHAPES_8B[layer]
    W = synthetic.weight(K, N, 0.02, 0.001, ("decode_8b", layer))
    _assert_exact(_gpu_quant(w4, W), W.numpy(), what=layer)


@pytest.mark.parametrize("layer", ["qkv", "down"])
def test_awq_exact(w4, layer):
    K, N = synthetic.SHAPES_8B[layer]
    W = synthetic.weight(K, N, 0.02, 0.0, ("verify_8b", layer))
    s = synthetic.awq_scale(K, ("verify_8b", layer))
    _assert_exact(_gpu_quant(w4, W, s), W.numpy(), s.numpy(), what=f"awq {layer}")


@pytest.mark.parametrize("layer", list(synthetic.SHAPES_70B))
def test_prefill_70b_layers_exact_sampled(w4, layer):
    """Full-size 70B layers quantized on the GPU; sampled rows checked exactly."""
    K, N = synthetic.SHAPES_70B[layer]
    tag = ("prefill_70b", layer)
    W = synthetic.weight(K, N, 0.015, 0.0, tag)
    packed, scales, zeros, codes = _gpu_quant(w4, W)
    rows = sample_rows(N, 48, seed=K + N)
    Wr = W[torch.from_numpy(rows)].numpy()
    _assert_exact((packed[rows], scales[rows], zeros[rows], codes[rows]), Wr, what=layer)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_16bit_weights_exact(w4, dtype):
    W = synthetic.weight(512, 300, 0.02, 0.001, ("w16", str(dtype))).to(dtype)
    _assert_exact(_gpu_quant(w4, W, dtype=dtype), W.float().numpy(), what=str(dtype))


@pytest.mark.parametrize("N,K", [(1, 128), (3, 256), (77, 384), (129, 1024)])
def test_ragged_shapes_exact(w4, N, K):
    W = synthetic.weight(K, N, 0.02, 0.01, ("ragged", N, K))
    _assert_exact(_gpu_quant(w4, W), W.numpy(), what=f"{N}x{K}")


def test_degenerate_and_tie_groups_exact(w4):
    rows = []
    rows.append(np.full(G, 3.0))                   # constant integer group
    rows.append(np.zeros(G))                       # zero group
    rows.append(np.full(G, -2.0))
    r = np.full(G, 0.5); r[5] = 0.5 + 1e-9; rows.append(r)  # fp16 scale underflows
    c = 2.0 ** -6
    r = np.zeros(G); r[0], r[1] = -7.5 * c, 7.5 * c; r[2:8] = [0.5 * c, -0.5 * c, 1.5 * c, 2.5 * c, -2.5 * c, 3 * c]
    rows.append(r)                                 # exact half-way ties
    rows.append(np.linspace(1.0, 2.0, G))          # group above zero (z clamps)
    rows.append(np.linspace(-3.0, -1.0, G))        # group below zero
    rng = np.random.default_rng(5)
    rows.append(rng.standard_normal(G) * 1e-6)     # subnormal fp16 scales
    rows.append(rng.standard_normal(G) * 3e3)      # large values
    W = torch.from_numpy(np.stack(rows).astype(np.float32))
    _assert_exact(_gpu_quant(w4, W), W.numpy(), what="special groups")
    s = torch.from_numpy(np.exp(rng.uniform(-3, 3, G)).astype(np.float32))
    _assert_exact(_gpu_quant(w4, W, s), W.numpy(), s.numpy(), what="special groups awq")


def test_pack_kernel_matches_oracle(w4):
    rng = np.random.default_rng(9)
    codes = rng.integers(0, 256, (37, 1024)).astype(np.uint8)  # values above 15 are masked
    packed = w4.w4_pack(torch.from_numpy(codes).cuda()).cpu().numpy()
    assert np.array_equal(packed, oracle.pack(codes))


def test_no_device_error(w4):
    assert w4.w4_device_error() == 0
