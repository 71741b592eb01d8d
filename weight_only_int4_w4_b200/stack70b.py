"""Whole-model 70B decode workload, built and run on one GPU.

The stack is 80 Llama-3-70B layers, each with four linear layers as (K, N):
qkv (8192, 10240), o_proj (8192, 8192), gate_up (8192, 57344) and
down (28672, 8192). lm_head (8192, 128256) comes last. That is 69.50 G
weights, or 36.92 GB once packed to uint4 with fp16 scales and zeros.

The dense fp32 weights of the whole stack (278 GB) do not fit on the device.
So each matrix is drawn on the device from a seeded CUDA generator, N(0, 0.015),
quantized there with ``w4_quantize`` and freed before the next one is drawn.
On request, a few rows of each dense matrix are first copied to the host so
that a checker can redo them on the CPU.

A decode step runs every linear layer once, in order, at M tokens. The
activations are synthetic, one bf16 N(0,1) matrix per input width K, so the
step measures the GEMMs alone.
"""
from __future__ import annotations

import numpy as np
import torch

from . import synthetic

STD = 0.015


def layer_list():
    """(index, name, K, N) of every linear layer of the stack, in execution order."""
    out = []
    for i in range(synthetic.N_LAYERS_70B):
        for name, (K, N) in synthetic.SHAPES_70B.items():
            out.append((i, name, K, N))
    K, N = synthetic.LM_HEAD_70B
    out.append((synthetic.N_LAYERS_70B, "lm_head", K, N))
    return out


def kept_rows(i, name, N, count):
    """Rows of matrix (i, name) copied to the host: the first, the last, and seeded others."""
    rng = np.random.default_rng(synthetic.seed_of("stack70b-rows", i, name) % (2 ** 32))
    rows = {0, N - 1}
    while len(rows) < count:
        rows.add(int(rng.integers(0, N)))
    return np.array(sorted(rows), dtype=np.int64)


def build(w4, keep=0, tag="stack70b"):
    """Draw, quantize and keep the packed stack on the current device.

    Returns (layers, quantize_ms, quantize_bytes). Each layer is a dict with
    K, N, packed, scales and zeros. With keep > 0 it also has rows (numpy) and
    W_rows (fp32 CPU tensor [len(rows), K]). quantize_ms is the summed device
    time of the quantize launches (their outputs are allocated before the
    timing events), and quantize_bytes is their algorithmic
    traffic: fp32 W in, plus packed codes, scales and zeros out.
    """
    gen = torch.Generator(device="cuda")
    layers = []
    q_ms, q_bytes = 0.0, 0
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i, name, K, N in layer_list():
        gen.manual_seed(synthetic.seed_of(tag, i, name) % (2 ** 62))
        W = torch.randn((N, K), generator=gen, device="cuda", dtype=torch.float32).mul_(STD)
        entry = dict(i=i, name=name, K=K, N=N)
        if keep:
            rows = kept_rows(i, name, N, keep)
            entry["rows"] = rows
            entry["W_rows"] = W[torch.from_numpy(rows).cuda()].cpu()
        # outputs are allocated before the first event, so only the launch is timed
        packed = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
        scales = torch.empty((N, K // 128), dtype=torch.float16, device="cuda")
        zeros = torch.empty((N, K // 128), dtype=torch.float16, device="cuda")
        a.record()
        w4.w4_quantize(W, out=(packed, scales, zeros))
        b.record()
        b.synchronize()
        q_ms += a.elapsed_time(b)
        q_bytes += 4 * N * K + N * K // 2 + 4 * N * (K // 128)
        del W
        entry.update(packed=packed, scales=scales, zeros=zeros)
        layers.append(entry)
    torch.cuda.synchronize()
    return layers, q_ms, q_bytes


def step_buffers(w4, layers, M, tag="stack70b"):
    """Activations (one per K), outputs (one per N) and one shared workspace for M tokens."""
    Ks = sorted({L["K"] for L in layers})
    Ns = sorted({L["N"] for L in layers})
    X = {K: synthetic.activations(M, K, "bf16", (tag, "X", M, K)).cuda() for K in Ks}
    Y = {N: torch.empty((M, N), dtype=torch.float32, device="cuda") for N in Ns}
    need = max(w4.w4a16_gemm_workspace_size(M, L["N"], L["K"]) for L in layers)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
    return X, Y, ws


def run_step(w4, layers, X, Y, ws, after_layer=None):
    """One decode step: every linear layer once, in order."""
    for L in layers:
        w4.w4a16_gemm(X[L["K"]], L["packed"], L["scales"], L["zeros"], out=Y[L["N"]], ws=ws)
        if after_layer is not None:
            after_layer(L, Y[L["N"]])


def step_bytes(layers, M):
    """Algorithmic bytes of one step: packed codes, scales, zeros, X (bf16) and Y (fp32) per layer."""
    return sum(L["N"] * L["K"] // 2 + 4 * L["N"] * (L["K"] // 128) + 2 * M * L["K"] + 4 * M * L["N"]
               for L in layers)
