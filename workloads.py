"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module draws random tensors and nothing else: it holds none of the FP8
linear layer's arithmetic (no scale formula, no rounding rule, no GEMM).  Both
the CUDA path and the CPU oracle consume what it returns, so the way a tensor is
drawn affects only the workload, never a parity comparison.

Distributions follow the workloads the AstrAI pages measure (a 12-layer,
dim-1024 transformer trained at batch 4 x 512 tokens; pre-quantized E4M3 GEMMs
on square, skinny and batched shapes):

* activations ``x ~ N(0, 1)``, weights ``w ~ N(0, 0.02)``, bias ``~ N(0, 0.1)``,
  output gradients ``g ~ N(0, 1e-3)``, each drawn in fp32 and rounded once to bf16;
* pre-quantized fp8 operands are N(0, 1) samples (optionally multiplied by a
  per-tensor factor) cast to fp8 by PyTorch's own dtype conversion, with GEMM
  scales drawn from U(0.5, 2);
* the delayed-scaling sequence multiplies ``x_t`` by ``s_t = 2^u``, ``u ~ U(-4, 4)``.

CPU generation uses ``torch.Generator().manual_seed(seed)``; ``device="cuda"``
uses a CUDA generator with the same seed (a different stream of numbers, used
only where the oracle samples the result instead of recomputing it whole).
"""

from __future__ import annotations

import math

import torch

# Training linears of a 12-layer dim-1024 transformer at B4 x T512: (K, N).
TRAINING_LINEARS = ((1024, 3072), (1024, 1024), (1024, 4096), (4096, 1024))
TRAINING_TOKENS = 2048
TRAINING_LAYERS = 12

SQUARE_SIZES = (512, 1024, 2048, 4096, 8192)

# (batch_a, batch_b, M, N, K): skinny and batched NT shapes.
SKINNY_BATCHED = ((1, 1, 64, 8192, 2048), (1, 1, 1024, 1536, 2048),
                  (64, 64, 512, 512, 512), (8, 1, 1024, 2048, 2048))


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """bf16 tensor of N(0, std^2) samples (drawn in fp32, rounded once)."""
    g = generator(seed, device)
    t = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    return (t * std).to(torch.bfloat16)


def uniform(lo: float, hi: float, seed: int, n: int = 1) -> torch.Tensor:
    g = generator(seed)
    return torch.rand(n, generator=g, dtype=torch.float32) * (hi - lo) + lo


def fp8_bytes(shape, seed: int, fmt: str = "e4m3", factor: float = 1.0,
              device="cpu") -> torch.Tensor:
    """uint8 tensor: N(0, 1) * factor samples cast to fp8 by PyTorch."""
    g = generator(seed, device)
    t = torch.randn(shape, generator=g, dtype=torch.float32, device=device) * factor
    dt = torch.float8_e4m3fn if fmt == "e4m3" else torch.float8_e5m2
    return t.to(dt).view(torch.uint8)


def amax_scaled_fp8_bytes(shape, seed: int, device="cpu"):
    """(uint8 E4M3 bytes, step): N(0,1) samples multiplied by 448/amax before the
    cast, and the matching step amax/448 for the GEMM."""
    g = generator(seed, device)
    t = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    a = float(t.abs().max())
    step = a / 448.0
    return (t * (448.0 / a)).to(torch.float8_e4m3fn).view(torch.uint8), step


def delayed_sequence_factors(steps: int = 8, seed: int = 0):
    """``s_t = 2^u_t``, ``u_t ~ U(-4, 4)``, one per step."""
    g = generator(seed)
    u = torch.rand(steps, generator=g, dtype=torch.float64) * 8.0 - 4.0
    return [math.pow(2.0, float(v)) for v in u]


def tiny_linear(seed: int = 0):
    """x [128,256] N(0,1), w [256,256] N(0,0.02), bias [256] N(0,0.1),
    g [128,256] N(0,1e-3), all bf16."""
    return dict(x=normal_bf16((128, 256), 1.0, seed),
                w=normal_bf16((256, 256), 0.02, seed + 1),
                b=normal_bf16((256,), 0.1, seed + 2),
                g=normal_bf16((128, 256), 1e-3, seed + 3))


def delayed_ring_inputs(step: int, factor: float, rows=512, cols=1024, seed=100):
    """x_t = bf16(N(0,1) * s_t) for one step of the delayed-scaling sequence."""
    g = generator(seed + step)
    t = torch.randn((rows, cols), generator=g, dtype=torch.float32) * factor
    return t.to(torch.bfloat16)


def training_linear(m: int, k: int, n: int, seed: int, device="cpu"):
    """One training linear: x [m,k], w [n,k], bias [n], g [m,n], bf16."""
    return dict(x=normal_bf16((m, k), 1.0, seed, device),
                w=normal_bf16((n, k), 0.02, seed + 1, device),
                b=normal_bf16((n,), 0.1, seed + 2, device),
                g=normal_bf16((m, n), 1e-3, seed + 3, device))


def bf16_bits(t: torch.Tensor):
    """numpy uint16 view of a CPU bf16 tensor (for the oracle)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")


def u8(t: torch.Tensor):
    """numpy uint8 view of a CPU byte tensor."""
    return t.contiguous().view(torch.uint8).numpy()
