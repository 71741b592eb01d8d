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


def test_static_scratch_wide_decode_shape_is_served_under_the_cap(w4, monkeypatch, capfd):
    """M=8 on the Llama-3-70B gate_up shape (8192 -> 57344): the decode kernel's
    k-slice partials would pass the fixed scratch, and the small-M tensor-core
    plan (or the prefill one) serves the call under the same cap.  Two calls in a
    row match w4a16_gemm with a caller-owned workspace, and the plan printed with
    W4_DEBUG_PLAN is not the decode kernel's."""
    M, N, K = 8, 57344, 8192
    assert w4.w4a16_gemm_workspace_size(M, N, K) > w4.w4a16_gemm_decode_static_capacity()
    tag = ("noalloc-wide", M, N, K)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(synthetic.seed_of(*tag) % (2 ** 62))
    W = torch.randn((N, K), generator=gen, device="cuda") * 0.015
    packed, scales, zeros = w4.w4_quantize(W)
    del W
    X = synthetic.activations(M, K, "bf16", tag).cuda()
    Yref = w4.w4a16_gemm(X, packed, scales, zeros)
    monkeypatch.setenv("W4_DEBUG_PLAN", "1")
    Y1 = w4.w4a16_gemm_decode_static(X, packed, scales, zeros)
    Y2 = w4.w4a16_gemm_decode_static(X, packed, scales, zeros)
    torch.cuda.synchronize()
    err = capfd.readouterr().err
    assert ("skinny" in err or "tensor-core" in err) and "decode:" not in err, err
    _check_sampled_and_all(w4, X, packed, scales, zeros, Yref, (Y1, Y2), "static scratch 70B gate_up M=8")
    del packed, scales, zeros
    torch.cuda.empty_cache()


def test_static_scratch_decode_plan_over_cap_falls_back_to_tensor_cores(w4, monkeypatch, capfd):
    """M=3 goes to the decode kernel at every shape; on 16384 -> 131072 its k-slice
    partials (3 slices x 2 slots x 3 x 131072 fp32, 9.4 MB) pass the fixed scratch,
    so the call takes the tensor-core plan under the same cap.  Random codes,
    scales and zero points (no quantization pass needed for a plan check)."""
    M, N, K = 3, 131072, 16384
    tag = ("noalloc-fallback", M, N, K)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(synthetic.seed_of(*tag) % (2 ** 62))
    packed = torch.randint(0, 256, (N, K // 2), generator=gen, device="cuda", dtype=torch.int32).to(torch.uint8)
    scales = (torch.rand((N, K // 128), generator=gen, device="cuda") * 0.002 + 1e-4).to(torch.float16)
    zeros = torch.randint(0, 16, (N, K // 128), generator=gen, device="cuda", dtype=torch.int32).to(torch.float16)
    X = synthetic.activations(M, K, "bf16", tag).cuda()
    Yref = w4.w4a16_gemm(X, packed, scales, zeros)
    monkeypatch.setenv("W4_DEBUG_PLAN", "1")
    Y1 = w4.w4a16_gemm_decode_static(X, packed, scales, zeros)
    Y2 = w4.w4a16_gemm_decode_static(X, packed, scales, zeros)
    torch.cuda.synchronize()
    err = capfd.readouterr().err
    assert "tensor-core" in err and "decode:" not in err, err
    _check_sampled_and_all(w4, X, packed, scales, zeros, Yref, (Y1, Y2), "static scratch M=3 fallback")
    del packed, scales, zeros
    torch.cuda.empty_cache()


def _check_sampled_and_all(w4, X, packed, scales, zeros, Yref, Ys, what):
    """Sampled rows against the oracle (from the library's own packed weights decoded
    on the host), and every output against w4a16_gemm: each is within
    2e-3 * sum_k |x w^| of the exact value, so the two differ by at most twice that
    (the sum formed here in plain torch)."""
    N, K = packed.shape[0], packed.shape[1] * 2
    rows = np.array([0, 1, N // 3, N // 2 + 7, N - 1])
    rsel = torch.from_numpy(rows).cuda()
    codes = oracle.unpack(packed[rsel].cpu().numpy(), K)
    What = oracle.dequant(codes, scales[rsel].cpu().numpy(), zeros[rsel].cpu().numpy())
    Yo, bound = oracle.gemm(X.float().cpu().numpy(), What)
    bound_all = torch.zeros((X.shape[0], N), dtype=torch.float64, device="cuda")
    for r0 in range(0, N, 16384):  # in row blocks, to bound the temporary
        pb = packed[r0:r0 + 16384]
        q = torch.stack([(pb & 15), (pb >> 4)], dim=-1).reshape(pb.shape[0], K).float()
        Wd = (q - zeros[r0:r0 + 16384].float().repeat_interleave(128, 1)) * \
            scales[r0:r0 + 16384].float().repeat_interleave(128, 1)
        bound_all[:, r0:r0 + 16384] = (X.float().abs() @ Wd.abs().t()).double()
        del q, Wd
    ref = Yref.cpu().numpy().astype(np.float64)
    bnd = bound_all.cpu().numpy()
    for Y in Ys:
        check_close(Y[:, rsel].cpu().numpy(), Yo, bound, what=what + " vs oracle")
        check_close(Y.cpu().numpy(), ref, 2.0 * bnd, what=what + " vs workspace entry")
    assert w4.w4_device_error() == 0


def test_static_scratch_rejects_oversized_forced_decode_plan(w4, monkeypatch):
    """With the decode kernel forced, a plan whose partials exceed the fixed
    scratch is rejected on the host with the sizes in the message."""
    M, N, K = 8, 65536, 8192
    monkeypatch.setenv("W4_FORCE_PATH", "gemv")
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
