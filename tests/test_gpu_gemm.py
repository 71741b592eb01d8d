"""GPU parity of the fused dequantize-matmul (K1 decode path, K3 skinny
tensor-core path, K2 tensor-core path) against the oracle: |y - y_ref| <= 2e-3 * sum_k |x w^| per element.

The weights given to the GPU GEMM are the ORACLE's packed codes, scales and
zeros (uploaded), so these tests check the matmul independently of K0; the
end-to-end tests at the bottom chain K0 -> GEMM."""
import os

import numpy as np
import pytest
import torch

import oracle
from weight_only_int4_w4_b200 import synthetic

from ._util import check_close, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    from weight_only_int4_w4_b200 import w4 as mod
    return mod


class forced_path:
    def __init__(self, path):
        self.path = path

    def __enter__(self):
        self.old = os.environ.get("W4_FORCE_PATH")
        if self.path:
            os.environ["W4_FORCE_PATH"] = self.path
        else:
            os.environ.pop("W4_FORCE_PATH", None)

    def __exit__(self, *a):
        if self.old is None:
            os.environ.pop("W4_FORCE_PATH", None)
        else:
            os.environ["W4_FORCE_PATH"] = self.old


def _upload_oracle_weights(W_np, awq_np=None):
    codes, scales, zeros = oracle.quantize(W_np, awq_np)
    packed = oracle.pack(codes)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return (dev(packed), dev(scales.view(np.uint16)).view(torch.float16), dev(zeros.view(np.uint16)).view(torch.float16),
            (codes, scales, zeros))


def _run_case(w4, M, N, K, x_dtype="bf16", awq=False, outliers=0.0, std=0.02, path=None, rows=None,
              out_dtype=torch.float32, tag=None):
    tag = tag or ("case", M, N, K, x_dtype, awq, outliers)
    W = synthetic.weight(K, N, std, outliers, tag)
    s = synthetic.awq_scale(K, tag) if awq else None
    X = synthetic.activations(M, K, x_dtype, tag)
    packed, scales, zeros, (codes, sc, zp) = _upload_oracle_weights(W.numpy(), None if s is None else s.numpy())
    with forced_path(path):
        Y = w4.w4a16_gemm(X.cuda(), packed, scales, zeros, None if s is None else s.cuda(), out_dtype=out_dtype)
    torch.cuda.synchronize()
    rows = np.arange(N) if rows is None else rows
    What = oracle.dequant(codes[rows], sc[rows], zp[rows], None if s is None else s.numpy())
    Yref, bound = oracle.gemm(X.float().numpy(), What)
    Yg = Y.float().cpu().numpy()[:, rows]
    return check_close(Yg, Yref, bound, out_bf16=out_dtype == torch.bfloat16, what=f"M={M} N={N} K={K} {path}")


def test_tiny_workload(w4):
    """256x256 fp32 weights, fp16 activations, M=1 (the oracle-sized case)."""
    _run_case(w4, 1, 256, 256, x_dtype="f16", tag=("tiny", "tiny"))


@pytest.mark.parametrize("layer", list(synthetic.SHAPES_8B))
def test_decode_8b_full(w4, layer):
    """M=1 bf16 decode at Llama-3-8B shapes with 0.1% outliers: every output checked."""
    K, N = synthetic.SHAPES_8B[layer]
    _run_case(w4, 1, N, K, outliers=0.001, tag=("decode_8b", layer))


@pytest.mark.parametrize("M", [4, 8, 16, 32, 48, 64])
@pytest.mark.parametrize("layer", list(synthetic.SHAPES_8B))
def test_verify_8b_awq_sampled(w4, M, layer):
    """Speculative-verification / small-batch M with the AWQ scale folded in."""
    K, N = synthetic.SHAPES_8B[layer]
    rows = sample_rows(N, 192, seed=M * 7 + K)
    _run_case(w4, M, N, K, awq=True, rows=rows, tag=("verify_8b", layer))


@pytest.mark.parametrize("layer", list(synthetic.SHAPES_70B))
def test_prefill_70b_sampled(w4, layer):
    """Prefill at Llama-3-70B shapes, M in {512, 2048, 8192}: sampled outputs of
    full-size launches, one weight quantization per layer reused for all M."""
    K, N = synthetic.SHAPES_70B[layer]
    tag = ("prefill_70b", layer)
    rows = sample_rows(N, 40, seed=K ^ N)
    Wr = synthetic.weight_rows(K, N, 0.015, 0.0, tag, rows=rows).numpy()
    # the GPU quantizes the full matrix itself (K0 is checked bit-exact elsewhere)
    W = synthetic.weight(K, N, 0.015, 0.0, tag).cuda()
    packed, scales, zeros = w4.w4_quantize(W)
    del W
    codes, sc, zp = oracle.quantize(Wr)
    What = oracle.dequant(codes, sc, zp)
    Xall = synthetic.activations(8192, K, "bf16", tag)
    for M in (512, 2048, 8192):
        X = Xall[:M]
        toks = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(M).choice(M, 24, replace=False)]))
        Y = w4.w4a16_gemm(X.cuda(), packed, scales, zeros)
        torch.cuda.synchronize()
        Yg = Y[torch.from_numpy(toks).cuda()][:, torch.from_numpy(rows).cuda()].float().cpu().numpy()
        del Y
        Yref, bound = oracle.gemm(X[torch.from_numpy(toks)].float().numpy(), What)
        check_close(Yg, Yref, bound, what=f"{layer} M={M}")


@pytest.mark.parametrize("path", ["gemv", "skinny", "tc"])
@pytest.mark.parametrize("M,N,K", [
    (1, 16, 128), (1, 1, 128), (2, 100, 256), (3, 129, 384), (7, 300, 1024), (9, 64, 128),
    (15, 200, 640), (17, 130, 256), (31, 77, 512), (33, 128, 1024), (63, 257, 256), (64, 320, 384),
])
def test_edge_shapes_both_paths(w4, M, N, K, path):
    _run_case(w4, M, N, K, path=path, tag=("edge", M, N, K))


@pytest.mark.parametrize("M,N,K", [(65, 300, 384), (100, 129, 1024), (129, 64, 256), (256, 513, 512),
                                   (300, 200, 1280)])
def test_edge_shapes_tc_only(w4, M, N, K):
    _run_case(w4, M, N, K, tag=("edge", M, N, K))


@pytest.mark.parametrize("path", ["gemv", "skinny", "tc"])
@pytest.mark.parametrize("x_dtype", ["f16", "bf16"])
def test_awq_and_dtypes(w4, path, x_dtype):
    _run_case(w4, 5, 384, 1024, x_dtype=x_dtype, awq=True, path=path, tag=("awq-dt", x_dtype))
    _run_case(w4, 24, 256, 512, x_dtype=x_dtype, awq=True, path=path, tag=("awq-dt24", x_dtype))


@pytest.mark.parametrize("path", ["gemv", "skinny", "tc"])
def test_bf16_output(w4, path):
    _run_case(w4, 4, 512, 1024, path=path, out_dtype=torch.bfloat16, tag=("bf16out",))


@pytest.mark.parametrize("M,N,K,awq,splits", [
    (21, 256, 2688, True, 5),    # AWQ kernel (8 dequant warps): one batch of 4 splits and 1 more
    (45, 384, 8192, False, 16),  # plain weights: four batches of 4 splits
    (13, 130, 3200, False, 6),   # one batch and 2 more, ragged weight rows
    (13, 130, 1536, False, 3),   # fewer splits than one batch
])
def test_split_k_reduction_ragged(w4, monkeypatch, capfd, M, N, K, awq, splits):
    """Tensor-core split-K: the last CTA of each tile sums the fp32 partials in
    batches of 4 splits plus a remainder, for token counts that are not multiples
    of 8.  The plan printed with W4_DEBUG_PLAN confirms the split count."""
    monkeypatch.setenv("W4_DEBUG_PLAN", "1")
    _run_case(w4, M, N, K, awq=awq, path="tc", tag=("splitk", M, N, K, awq))
    err = capfd.readouterr().err
    assert f"tensor-core: bn=64 splits={splits} " in err, err


@pytest.mark.parametrize("M,N,K,awq,out,bn,tiles,pieces", [
    (300, 9688, 4096, False, "f32", 256, 152, 4),    # 4 tail tiles in 4 pieces, ragged last n-tile and tokens
    (300, 9688, 3200, True, "bf16", 256, 152, 3),    # AWQ kernel, uneven last piece, bf16 output
    (100, 38149, 5120, False, "f32", 128, 299, 5),  # two CTAs per SM (296 slots): one batch of 4 pieces + 1
])
def test_tail_split_last_wave(w4, monkeypatch, capfd, M, N, K, awq, out, bn, tiles, pieces):
    """Tensor-core tail split: whole tiles fill complete waves and the last,
    mostly empty wave's tiles are cut along K; the reduction kernel sums the
    pieces.  Every output of the tail tiles is checked, with a sample elsewhere."""
    monkeypatch.setenv("W4_DEBUG_PLAN", "1")
    ntx = (N + 127) // 128
    slots = 148 * (1 if (awq or bn == 256) else 2)
    head = tiles - tiles % slots
    tail_rows = set()
    for t in range(head, tiles):
        n0 = (t % ntx) * 128
        tail_rows.update(range(n0, min(n0 + 128, N)))
    rows = np.array(sorted(tail_rows | set(sample_rows(N, 48, seed=N ^ K).tolist())))
    _run_case(w4, M, N, K, awq=awq, path="tc", rows=rows,
              out_dtype=torch.bfloat16 if out == "bf16" else torch.float32, tag=("tail", M, N, K, awq))
    err = capfd.readouterr().err
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert f"bn={bn} splits=1 " in err and f"head_tiles={head} tail_pieces={pieces} " in err, err


@pytest.mark.parametrize("M,N,K,out", [
    (200, 1000, 512, "bf16"),  # ragged tokens (last 32-token box partly past M), last 128-row tile partly past N
    (200, 904, 512, "f32"),    # the last tile's second 32-row box starts past N and is skipped
    (33, 904, 512, "bf16"),    # one token past a 32-token box
])
def test_tma_store_epilogue_ragged(w4, monkeypatch, capfd, M, N, K, out):
    """Tensor-core tiles written by 32 x 32 TMA stores (Y rows are 16-byte
    multiples, M and N >= 32, one split): the stores clip at M and N, and
    every output is checked."""
    monkeypatch.setenv("W4_DEBUG_PLAN", "1")
    _run_case(w4, M, N, K, path="tc", out_dtype=torch.bfloat16 if out == "bf16" else torch.float32,
              tag=("tma-store", M, N, K, out))
    err = capfd.readouterr().err
    assert "splits=1 " in err and "tail_pieces=0 " in err, err


def test_long_k_split_both_paths(w4):
    """K = 28672 (70B down_proj depth) at small M: split-K on both paths."""
    for path in ("gemv", "skinny", "tc"):
        _run_case(w4, 2, 512, 28672, path=path, tag=("longk",))


def test_workspace_reuse_is_stable(w4):
    """Split-K counters are left at zero: repeated calls give identical bits."""
    K, N = 14336, 4096
    tag = ("reuse",)
    W = synthetic.weight(K, N, 0.02, 0.0, tag).cuda()
    packed, scales, zeros = w4.w4_quantize(W)
    X = synthetic.activations(1, K, "bf16", tag).cuda()
    for path in ("gemv", "skinny", "tc"):
        with forced_path(path):
            outs = [w4.w4a16_gemm(X, packed, scales, zeros).clone() for _ in range(3)]
        torch.cuda.synchronize()
        assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


def test_end_to_end_quantize_then_gemm(w4):
    """K0 on the GPU feeding the GEMM, against the oracle's whole path."""
    M, N, K = 3, 1000, 4096
    tag = ("e2e",)
    W = synthetic.weight(K, N, 0.02, 0.001, tag)
    s = synthetic.awq_scale(K, tag)
    X = synthetic.activations(M, K, "bf16", tag)
    packed, scales, zeros = w4.w4_quantize(W.cuda(), s.cuda())
    Y = w4.w4a16_gemm(X.cuda(), packed, scales, zeros, s.cuda())
    Yref, bound, _ = oracle.reference_linear(X.float().numpy(), W.numpy(), s.numpy())
    check_close(Y.cpu().numpy(), Yref, bound, what="e2e")


def test_host_entry_point(w4):
    M, N, K = 2, 640, 2048
    tag = ("host",)
    W = synthetic.weight(K, N, 0.02, 0.0, tag)
    X = synthetic.activations(M, K, "bf16", tag)
    packed, scales, zeros = w4.w4_quantize(W.cuda())
    Xh = X.pin_memory()
    Yh = torch.empty((M, N), dtype=torch.float32).pin_memory()
    w4.w4a16_gemm_host(Xh, torch.empty_like(X, device="cuda"), packed, scales, zeros, Yh,
                       torch.empty((M, N), dtype=torch.float32, device="cuda"))
    Yref, bound, _ = oracle.reference_linear(X.float().numpy(), W.numpy())
    check_close(Yh.numpy(), Yref, bound, what="host")


def test_host_entry_point_async_waits_once(w4):
    """Two layers through w4a16_gemm_host_async on one stream, one wait at the end:
    both host outputs match the oracle (and the per-call-wait entry's results)."""
    stream = torch.cuda.Stream()
    outs = []
    for i, (M, N, K) in enumerate(((1, 640, 2048), (3, 1024, 4096))):
        tag = ("host-async", i)
        W = synthetic.weight(K, N, 0.02, 0.0, tag)
        X = synthetic.activations(M, K, "bf16", tag)
        packed, scales, zeros = w4.w4_quantize(W.cuda())
        torch.cuda.synchronize()
        Xh = X.pin_memory()
        Yh = torch.full((M, N), float("nan"), dtype=torch.float32).pin_memory()
        Yd = torch.empty((M, N), dtype=torch.float32, device="cuda")
        w4.w4a16_gemm_host(Xh, torch.empty_like(X, device="cuda"), packed, scales, zeros, Yh, Yd, stream=stream,
                           wait=False)
        outs.append((Yh, X, W, (packed, scales, zeros, Yd)))
    stream.synchronize()
    for Yh, X, W, keep in outs:
        Yref, bound, _ = oracle.reference_linear(X.float().numpy(), W.numpy())
        check_close(Yh.numpy(), Yref, bound, what="host async")


def test_host_batch_entry_matches_the_oracle_and_single_calls(w4):
    """Four independent matmuls through w4a16_gemm_host_batch_async (one copy in,
    the matmuls, one copy out, one wait): decode, small-M and prefill shapes, f16
    and bf16 activations, fp32 and bf16 outputs, one with AWQ.  Each output matches
    the oracle and, bit for bit, the same matmul through w4a16_gemm."""
    cases = [(1, 640, 2048, "bf16", torch.float32, False), (5, 384, 1024, "f16", torch.bfloat16, True),
             (24, 512, 1024, "bf16", torch.float32, False), (300, 256, 512, "bf16", torch.bfloat16, False)]
    items, keep, xo, yo = [], [], 0, 0
    for i, (M, N, K, xd, yd, awq) in enumerate(cases):
        tag = ("host-batch", i)
        W = synthetic.weight(K, N, 0.02, 0.0, tag)
        s = synthetic.awq_scale(K, tag) if awq else None
        X = synthetic.activations(M, K, xd, tag)
        packed, scales, zeros, (codes, sc, zp) = _upload_oracle_weights(W.numpy(), None if s is None else s.numpy())
        s_dev = None if s is None else s.cuda()
        items.append(dict(M=M, N=N, K=K, packed=packed, scales=scales, zeros=zeros, awq_s=s_dev, x_offset=xo,
                          y_offset=yo, x_dtype=X.dtype, y_dtype=yd))
        keep.append((X, s, s_dev, codes, sc, zp, xo, yo, yd))
        xo += -(-M * K * 2 // 16) * 16
        yo += -(-M * N * (4 if yd == torch.float32 else 2) // 16) * 16
    Xh = torch.zeros(xo, dtype=torch.uint8).pin_memory()
    for (X, *_rest), it in zip(keep, items):
        Xh[it["x_offset"]:it["x_offset"] + X.numel() * 2] = X.contiguous().view(torch.uint8).reshape(-1)
    Yh = torch.full((yo,), 0xFF, dtype=torch.uint8).pin_memory()
    Xd = torch.empty(xo, dtype=torch.uint8, device="cuda")
    Yd = torch.empty(yo, dtype=torch.uint8, device="cuda")
    need = max(w4.w4a16_gemm_workspace_size(it["M"], it["N"], it["K"]) for it in items)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    w4.w4a16_gemm_host_batch(w4.gemm_batch(items), Xh, Xd, Yh, Yd, ws=ws, stream=stream, wait=True)
    for (X, s, s_dev, codes, sc, zp, xo_i, yo_i, yd), it in zip(keep, items):
        M, N = it["M"], it["N"]
        nb = M * N * (4 if yd == torch.float32 else 2)
        Yb = Yh[yo_i:yo_i + nb].view(yd).reshape(M, N)
        What = oracle.dequant(codes, sc, zp, None if s is None else s.numpy())
        Yref, bound = oracle.gemm(X.float().numpy(), What)
        check_close(Yb.float().numpy(), Yref, bound, out_bf16=yd == torch.bfloat16, what=f"batch M={M}")
        Y1 = w4.w4a16_gemm(X.cuda(), it["packed"], it["scales"], it["zeros"], s_dev, out_dtype=yd)
        torch.cuda.synchronize()
        assert torch.equal(Y1.cpu().view(torch.uint8), Yb.view(torch.uint8)), f"batch M={M}: not the single-call bits"


def test_short_workspace_rejected(w4):
    M, N, K = 1, 4096, 14336
    need = w4.w4a16_gemm_workspace_size(M, N, K)
    assert need > 0
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((N, K // 128), dtype=torch.float16, device="cuda")
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")  # far below any split-K plan's need
    with pytest.raises(w4.W4Error) as ei:
        w4.w4a16_gemm(X, packed, sc, sc, ws=small)
    assert ei.value.status == w4.W4_ERR_INVALID_ARG


def test_no_device_error(w4):
    assert w4.w4_device_error() == 0


def _degenerate_layer(N, K, seed):
    """Weights holding the method's degenerate groups among ordinary rows: all-zero
    rows, constant-integer groups, constant non-integer groups, all-positive and
    all-negative groups (the zero point clamps to 0 or 15), and a group with a
    single non-zero weight (every other code equals the zero point)."""
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    G = 128
    Kg = K // G
    W[0:4] = 0.0
    W[4] = np.repeat((np.arange(Kg) % 7 - 3).astype(np.float32), G)[:K]
    W[5] = 0.37
    W[6] = rng.uniform(0.5, 1.0, K)
    W[7] = rng.uniform(-1.0, -0.5, K)
    W[8] = 0.0
    W[8, 5::G] = 0.9
    W[9, :G] = 0.0  # one zero group inside an ordinary row
    W[N - 1] = 0.0  # a zero row in the ragged last tile
    return W


@pytest.mark.parametrize("path", ["gemv", "skinny", "tc"])
@pytest.mark.parametrize("M", [1, 8, 64])
@pytest.mark.parametrize("awq", [False, True])
def test_degenerate_weights_both_paths(w4, path, M, awq):
    """Degenerate weight groups through both GEMM kernels, with one token of
    large same-sign activations (every x = +1000): element-wise against the
    oracle at the accuracy bar, and rows of zero weights give exactly 0 (their
    bound sum_k |x w^| is 0)."""
    N, K = 200, 1024
    W = _degenerate_layer(N, K, seed=M + 100 * awq)
    s = synthetic.awq_scale(K, ("degenerate", M)).numpy() if awq else None
    X = synthetic.activations(M, K, "bf16", ("degenerate", M, awq))
    X[0] = 1000.0
    packed, scales, zeros, (codes, sc, zp) = _upload_oracle_weights(W, s)
    with forced_path(path):
        Y = w4.w4a16_gemm(X.cuda(), packed, scales, zeros, None if s is None else torch.from_numpy(s).cuda())
    torch.cuda.synchronize()
    What = oracle.dequant(codes, sc, zp, s)
    Yref, bound = oracle.gemm(X.float().numpy(), What)
    Yg = Y.cpu().numpy()
    zero_rows = [0, 1, 2, 3, N - 1]
    assert np.all(bound[:, zero_rows] == 0.0)
    assert np.all(Yg[:, zero_rows] == 0.0), f"{path} M={M}: zero rows give {Yg[:, zero_rows].max()}"
    check_close(Yg, Yref, bound, what=f"degenerate {path} M={M} awq={awq}")


@pytest.mark.parametrize("path", ["gemv", "skinny", "tc"])
def test_back_to_back_calls_share_workspace(w4, path):
    """Four calls queued on one stream with one workspace and different
    activations, no synchronization between them: each call's staged
    activations and split-K partials must not be touched by the next call
    before it is done (programmatic launches wait for their predecessor)."""
    M, N, K = 24, 640, 2048
    tag = ("b2b", path)
    W = synthetic.weight(K, N, 0.02, 0.0, tag)
    packed, scales, zeros, (codes, sc, zp) = _upload_oracle_weights(W.numpy())
    Xs = [synthetic.activations(M, K, "bf16", tag + (i,)) for i in range(4)]
    ws = torch.zeros(w4.w4a16_gemm_workspace_size(M, N, K) + 16, dtype=torch.uint8, device="cuda")
    with forced_path(path):
        Ys = [w4.w4a16_gemm(X.cuda(), packed, scales, zeros, ws=ws) for X in Xs]
    torch.cuda.synchronize()
    What = oracle.dequant(codes, sc, zp)
    for i, (X, Y) in enumerate(zip(Xs, Ys)):
        Yref, bound = oracle.gemm(X.float().numpy(), What)
        check_close(Y.cpu().numpy(), Yref, bound, what=f"back-to-back {path} call {i}")
