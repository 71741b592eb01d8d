"""Shared helpers of the GPU parity tests: seeded inputs, the oracle's answers,
and the element-wise tolerance check.  The oracle is only called from here and
from the tests."""
import numpy as np
import torch

import oracle
from weight_only_int4_w4_b200 import synthetic

G = 128
TOL = 2e-3  # |y - y_ref| <= TOL * sum_k |x w^| per element


def oracle_quant(W_np, awq_np=None):
    codes, scales, zeros = oracle.quantize(W_np, awq_np)
    return codes, scales, zeros


def to_np_f32(t):
    return t.detach().float().cpu().numpy()


def check_close(Y_gpu, Y_ref, bound, out_bf16=False, what=""):
    """Element-wise bar: |y - y_ref| <= 2e-3 * sum_k |x w^| (plus bf16 output rounding)."""
    Y_gpu = np.asarray(Y_gpu, np.float64)
    err = np.abs(Y_gpu - Y_ref)
    tol = TOL * bound + (2.0 ** -8) * np.abs(Y_ref) * (1 if out_bf16 else 0) + 1e-30
    ratio = err / tol
    worst = float(ratio.max()) if ratio.size else 0.0
    assert np.all(np.isfinite(Y_gpu)), f"{what}: non-finite output"
    assert worst <= 1.0, f"{what}: worst err/tol = {worst:.3g} at {np.unravel_index(np.argmax(ratio), ratio.shape)}"
    return worst


def sample_rows(N, count, seed):
    rng = np.random.default_rng(seed)
    base = {0, N - 1, min(127, N - 1), min(128, N - 1), N // 2}
    extra = rng.choice(N, size=min(count, N), replace=False)
    return np.array(sorted(base | set(int(v) for v in extra)))
