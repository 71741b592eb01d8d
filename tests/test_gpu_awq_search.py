"""GPU parity of the AWQ exponent search (w4_awq_search) against the oracle's
plain-loop search.

The error of each exponent must agree with the oracle's fp64 error within 2%.
The GPU's quantized products round W^ to bf16 once; that moves the error by a
few 1e-4 relative. The exponent the GPU picks must be optimal within that 2%
on the oracle's errors. The returned s must equal, to 1 ulp, the oracle's
s = m^a for that exponent.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_int4_w4_b200 import synthetic

pytestmark = pytest.mark.gpu

ALPHAS = [-1.0, -0.8, -0.6, -0.4, -0.2, 0.0, 0.2, 0.4, 0.6, 0.8, 1.0]


@pytest.fixture(scope="module")
def w4():
    from weight_only_int4_w4_b200 import w4 as mod
    return mod


def _calibration(Mc, K, tag):
    """bf16 N(0,1) calibration activations with 1% of the channels x10 (heavy channels)."""
    g = torch.Generator().manual_seed(synthetic.seed_of(tag, "calib") % (2 ** 62))
    X = torch.randn((Mc, K), generator=g)
    heavy = torch.randperm(K, generator=g)[: max(1, round(0.01 * K))]
    X[:, heavy] *= 10.0
    return X.to(torch.bfloat16)


@pytest.mark.parametrize("N,K,Mc,group", [(256, 512, 128, 128), (192, 1024, 64, 64), (64, 256, 96, 32)])
def test_awq_search_matches_oracle(w4, N, K, Mc, group):
    tag = ("awq-search", N, K, Mc, group)
    W = synthetic.weight(K, N, 0.02, 0.001, tag)
    X = _calibration(Mc, K, tag)
    s_gpu, a_gpu, errs = w4.w4_awq_search(W.cuda(), X.cuda(), ALPHAS, group=group)
    torch.cuda.synchronize()
    e_ref, s_ref, best_ref = oracle.awq_search(W.numpy(), X.float().numpy(), ALPHAS, group=group)
    errs = np.array(errs)
    assert np.all(np.abs(errs - e_ref) <= 2e-2 * e_ref), (errs, e_ref)
    i = ALPHAS.index(a_gpu)
    assert e_ref[i] <= e_ref.min() * (1 + 2e-2)
    # s for the GPU's exponent, from the oracle (same exponent -> same formula)
    _, s_i, _ = oracle.awq_search(W.numpy()[:1], X.float().numpy(), [a_gpu], group=group)
    sg = s_gpu.cpu().numpy()
    ulp = np.spacing(np.abs(s_i).astype(np.float32))
    assert np.all(np.abs(sg - s_i) <= ulp), "s differs by more than 1 ulp"
    # the heavy channels get s < 1 when a negative exponent wins
    if a_gpu < 0:
        assert sg.min() < 1.0


def test_awq_search_beats_plain_rtn_with_heavy_channels(w4):
    """With 1% heavy channels, the best exponent has a smaller output error than a = 0 (plain RTN)."""
    W = synthetic.weight(1024, 512, 0.02, 0.0, ("awq-gain",))
    X = _calibration(256, 1024, ("awq-gain",))
    _, a, errs = w4.w4_awq_search(W.cuda(), X.cuda(), ALPHAS)
    assert errs[ALPHAS.index(a)] < errs[ALPHAS.index(0.0)]


def test_no_device_error(w4):
    assert w4.w4_device_error() == 0
