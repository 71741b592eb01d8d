"""Seeded synthetic inputs for the W4A16 linear layers (no quantization arithmetic here).

Both the CUDA path and the CPU oracle are fed from these generators; this
module holds nothing of the method itself (no min/max, scale, zero, rounding or
matmul).  Every tensor is drawn on the CPU from a ``torch.Generator`` seeded by
a stable hash of (workload, layer, role), so any process can regenerate it.

Weights are drawn in blocks of ``ROW_BLOCK`` output rows, each block with its
own seed, so a sampled subset of rows of a very large matrix can be regenerated
without drawing the whole matrix.

Workload shapes (Llama-3-8B and Llama-3-70B linear layers, as (K, N) =
(input channels, output channels)):
  8B : qkv (4096, 6144), o_proj (4096, 4096), gate_up (4096, 28672), down (14336, 4096)
  70B: qkv (8192, 10240), o_proj (8192, 8192), gate_up (8192, 57344), down (28672, 8192),
       lm_head (8192, 128256)
"""
from __future__ import annotations

import zlib

import numpy as np
import torch

ROW_BLOCK = 128

SHAPES_8B = {"qkv": (4096, 6144), "o_proj": (4096, 4096), "gate_up": (4096, 28672), "down": (14336, 4096)}
SHAPES_70B = {"qkv": (8192, 10240), "o_proj": (8192, 8192), "gate_up": (8192, 57344), "down": (28672, 8192)}
LM_HEAD_70B = (8192, 128256)
N_LAYERS_70B = 80

# Workload catalogue.  Distribution parameters are standard deviations.
WORKLOADS = {
    "tiny": dict(shapes={"tiny": (256, 256)}, Ms=[1], x_dtype="f16", w_std=0.02,
                 outlier_frac=0.0, awq=False),
    "decode_8b": dict(shapes=SHAPES_8B, Ms=[1], x_dtype="bf16", w_std=0.02,
                      outlier_frac=0.001, awq=False),
    "verify_8b": dict(shapes=SHAPES_8B, Ms=[4, 8, 16, 32, 48, 64], x_dtype="bf16", w_std=0.02,
                      outlier_frac=0.0, awq=True),
    "prefill_70b": dict(shapes=SHAPES_70B, Ms=[512, 2048, 8192], x_dtype="bf16", w_std=0.015,
                        outlier_frac=0.0, awq=False),
}
OUTLIER_STD = 0.4


def seed_of(*parts) -> int:
    """Stable 63-bit seed from a tuple of names/numbers."""
    key = "/".join(str(p) for p in parts).encode()
    return (zlib.crc32(key) * 2654435761 + zlib.adler32(key)) % (2 ** 63 - 1)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def weight_rows(K: int, N: int, std: float, outlier_frac: float, tag, rows=None) -> torch.Tensor:
    """fp32 weight rows [len(rows), K] of the [N, K] matrix named by ``tag``.

    Entries are N(0, std); with ``outlier_frac`` > 0 each entry is, with that
    probability, replaced by a fresh N(0, 0.4) draw (symmetric outliers).
    ``rows`` = None returns all N rows.
    """
    rows = np.arange(N) if rows is None else np.asarray(rows)
    out = torch.empty((len(rows), K), dtype=torch.float32)
    blocks = np.unique(rows // ROW_BLOCK)
    for b in blocks:
        r0 = int(b) * ROW_BLOCK
        nb = min(ROW_BLOCK, N - r0)
        g = _gen(seed_of(tag, "W", K, N, int(b)))
        blk = torch.randn((nb, K), generator=g, dtype=torch.float32) * std
        if outlier_frac > 0:
            mask = torch.rand((nb, K), generator=g) < outlier_frac
            vals = torch.randn((nb, K), generator=g, dtype=torch.float32) * OUTLIER_STD
            blk = torch.where(mask, vals, blk)
        sel = np.nonzero((rows >= r0) & (rows < r0 + nb))[0]
        out[torch.from_numpy(sel)] = blk[torch.from_numpy(rows[sel] - r0)]
    return out


def weight(K: int, N: int, std: float, outlier_frac: float, tag) -> torch.Tensor:
    return weight_rows(K, N, std, outlier_frac, tag)


def activations(M: int, K: int, dtype: str, tag) -> torch.Tensor:
    """Activations X [M, K], N(0, 1), rounded to fp16 or bf16."""
    g = _gen(seed_of(tag, "X", M, K))
    x = torch.randn((M, K), generator=g, dtype=torch.float32)
    return x.to(torch.float16 if dtype == "f16" else torch.bfloat16)


def awq_scale(K: int, tag, calib_rows: int = 512, heavy_frac: float = 0.01, heavy_gain: float = 10.0) -> torch.Tensor:
    """Per-input-channel activation magnitude s [K] (fp32) from a seeded calibration batch.

    The calibration activations are a [512, K] N(0,1) matrix in which
    round(0.01 K) channels (chosen by the same generator) are multiplied by 10;
    s_k = (mean over rows of |c_k|) ** 0.5, computed in fp64 then rounded to
    fp32.  The vector is an input of the quantizer and of the matmul.
    """
    g = _gen(seed_of(tag, "awq_calib", K))
    c = torch.randn((calib_rows, K), generator=g, dtype=torch.float64)
    n_heavy = int(round(heavy_frac * K))
    heavy = torch.randperm(K, generator=g)[:n_heavy]
    c[:, heavy] *= heavy_gain
    s = c.abs().mean(dim=0).sqrt()
    return s.to(torch.float32)
