"""Short launch sequences of each kernel, for Nsight Compute captures.

    python -m weight_only_int4_w4_b200.profile_cases <case>

Cases (seeded synthetic inputs drawn on the device, bf16 activations):
  decode_step       the decode_8b step -- qkv 4096->6144, o_proj 4096->4096,
                    gate_up 4096->28672, down 14336->4096 at M=1 -- 4 times
  gemv_gate_up      gate_up 4096->28672 at M=1, 4 launches
  tc_o_proj         Llama-3-70B o_proj 8192->8192 at M=2048, 3 launches
  tc_awq_gate_up    gate_up 4096->28672 with AWQ scales at M=48 (speculative
                    verification of 8 drafts x 6 tokens), 3 launches
  skinny_gate_up    gate_up 4096->28672 with AWQ scales at M=16 on the skinny
                    tensor-core kernel (staging kernel + matmul), 3 launches
  quantize_gate_up  quantize+pack of gate_up's fp32 weights, 3 launches

Each case launches eagerly (no CUDA graph), checks the device error word and
prints one line.  It times nothing: the numbers come from the profiler.
"""
from __future__ import annotations

import os
import sys

import torch

from . import synthetic, w4

CASES = ("decode_step", "gemv_gate_up", "tc_o_proj", "tc_awq_gate_up", "skinny_gate_up", "quantize_gate_up")


def _weights(K, N, std, gen):
    W = torch.randn((N, K), generator=gen, device="cuda") * std
    packed, scales, zeros = w4.w4_quantize(W)
    return W, packed, scales, zeros


def run(case: str) -> None:
    if case not in CASES:
        raise SystemExit(f"unknown case {case!r}; one of {', '.join(CASES)}")
    torch.cuda.set_device(0)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(synthetic.seed_of("profile", case) % (2 ** 62))
    if case == "decode_step":
        layers = []
        for name, (K, N) in synthetic.SHAPES_8B.items():
            W, packed, scales, zeros = _weights(K, N, 0.02, gen)
            del W
            X = torch.randn((1, K), generator=gen, device="cuda").to(torch.bfloat16)
            layers.append((X, packed, scales, zeros, torch.empty((1, N), device="cuda")))
        for _ in range(4):
            for X, packed, scales, zeros, Y in layers:
                w4.w4a16_gemm(X, packed, scales, zeros, out=Y)
    elif case == "gemv_gate_up":
        K, N = synthetic.SHAPES_8B["gate_up"]
        W, packed, scales, zeros = _weights(K, N, 0.02, gen)
        del W
        X = torch.randn((1, K), generator=gen, device="cuda").to(torch.bfloat16)
        Y = torch.empty((1, N), device="cuda")
        for _ in range(4):
            w4.w4a16_gemm(X, packed, scales, zeros, out=Y)
    elif case == "tc_o_proj":
        K, N = synthetic.SHAPES_70B["o_proj"]
        W, packed, scales, zeros = _weights(K, N, 0.015, gen)
        del W
        X = torch.randn((2048, K), generator=gen, device="cuda").to(torch.bfloat16)
        Y = torch.empty((2048, N), device="cuda")
        for _ in range(3):
            w4.w4a16_gemm(X, packed, scales, zeros, out=Y)
    elif case == "tc_awq_gate_up":
        K, N = synthetic.SHAPES_8B["gate_up"]
        s = synthetic.awq_scale(K, ("profile", case)).cuda()
        W = torch.randn((N, K), generator=gen, device="cuda") * 0.02
        packed, scales, zeros = w4.w4_quantize(W, awq_s=s)
        del W
        X = torch.randn((48, K), generator=gen, device="cuda").to(torch.bfloat16)
        Y = torch.empty((48, N), device="cuda")
        for _ in range(3):
            w4.w4a16_gemm(X, packed, scales, zeros, awq_s=s, out=Y)
    elif case == "skinny_gate_up":
        K, N = synthetic.SHAPES_8B["gate_up"]
        s = synthetic.awq_scale(K, ("profile", case)).cuda()
        W = torch.randn((N, K), generator=gen, device="cuda") * 0.02
        packed, scales, zeros = w4.w4_quantize(W, awq_s=s)
        del W
        X = torch.randn((16, K), generator=gen, device="cuda").to(torch.bfloat16)
        Y = torch.empty((16, N), device="cuda")
        os.environ["W4_FORCE_PATH"] = "skinny"
        for _ in range(3):
            w4.w4a16_gemm(X, packed, scales, zeros, awq_s=s, out=Y)
        os.environ.pop("W4_FORCE_PATH")
    else:
        K, N = synthetic.SHAPES_8B["gate_up"]
        W = torch.randn((N, K), generator=gen, device="cuda") * 0.02
        for _ in range(3):
            w4.w4_quantize(W)
    torch.cuda.synchronize()
    err = w4.w4_device_error()
    print(f"{case}: done, device error word {err}")
    if err:
        raise SystemExit(1)


if __name__ == "__main__":
    run(sys.argv[1] if len(sys.argv) > 1 else "")
