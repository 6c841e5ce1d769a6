"""Seeded synthetic bf16 inputs for the five workloads of the scaled FP8 GEMM.

This module only draws random numbers.  It holds none of the quantization or
GEMM arithmetic, and it serves the tests, the benchmark and the CPU oracle
alike (the oracle reads the same bf16 bytes; it never regenerates them).

Recipe: ``g = torch.Generator('cpu').manual_seed(seed)``.  Draw fp32
``randn * sigma`` in a fixed order (A, then B, then the outlier choices),
scale the outliers in fp32, then cast to bfloat16 (round to nearest even).

Shapes follow the pages:
* ``tiny``    M=128,N=256,K=512, per-token mode.  The small DeepGEMM-style case.
* ``qk``      M=2048 (batch 2 x seq 1024), N=1024, K=4096, MX mode.  The Q.K^T
  example of the fp8_gemm listing on the "从 DeepGEMM 到 vLLM" page.  One percent
  of A's rows and of B's columns are scaled x50 as outliers.
* ``attn``    M=8192, N=2048, K=8192, per-token mode.  The first
  ``benchmark_gemm`` shape on the same page.
* ``ffn_up``  M=8192, N=22016, K=8192, MX mode.  The second ``benchmark_gemm``
  shape (FFN up-projection).  Weights are N(0, 0.02^2) with 0.1 % elementwise
  outliers x20.
* ``decode``  M in {1, 8, 32, 64} against Llama-3-8B-sized linears, MX mode.
  Shapes: up/gate 14336x4096, down 4096x14336, fused QKV 6144x4096.  Weights
  are N(0, 0.02^2).

B is returned in the layout the library takes: [N, K] with K contiguous
(B^T of the pages' logical [K, N]).
"""
from __future__ import annotations

import torch

DECODE_SHAPES = {"up": (14336, 4096), "down": (4096, 14336), "qkv": (6144, 4096)}
DECODE_M = (1, 8, 32, 64)

CONFIGS = {
    "tiny": dict(mode="rowwise", M=128, N=256, K=512, seed=0),
    "qk": dict(mode="mx", M=2048, N=1024, K=4096, seed=1),
    "attn": dict(mode="rowwise", M=8192, N=2048, K=8192, seed=2),
    "ffn_up": dict(mode="mx", M=8192, N=22016, K=8192, seed=3),
    "decode": dict(mode="mx", seed=4),
}


def _gen(seed: int) -> torch.Generator:
    return torch.Generator(device="cpu").manual_seed(seed)


def randn_bf16(shape, g: torch.Generator, sigma: float = 1.0) -> torch.Tensor:
    return (torch.randn(shape, generator=g, dtype=torch.float32) * sigma).to(torch.bfloat16)


def tiny():
    """A [128,512], B^T [256,512]; N(0,1), seed 0."""
    g = _gen(0)
    a = torch.randn((128, 512), generator=g, dtype=torch.float32)
    b = torch.randn((512, 256), generator=g, dtype=torch.float32)
    return a.to(torch.bfloat16), b.t().contiguous().to(torch.bfloat16)


def qk():
    """A [2048,4096], B^T [1024,4096]; N(0,1); 20 rows of A and 10 columns of the
    logical B [K,N] (rows of B^T) scaled x50, chosen without replacement; seed 1."""
    g = _gen(1)
    a = torch.randn((2048, 4096), generator=g, dtype=torch.float32)
    b = torch.randn((4096, 1024), generator=g, dtype=torch.float32)
    rows = torch.randperm(2048, generator=g)[:20]
    cols = torch.randperm(1024, generator=g)[:10]
    a[rows] *= 50.0
    b[:, cols] *= 50.0
    return a.to(torch.bfloat16), b.t().contiguous().to(torch.bfloat16)


def attn():
    """A [8192,8192], B^T [2048,8192]; N(0,1); seed 2."""
    g = _gen(2)
    a = torch.randn((8192, 8192), generator=g, dtype=torch.float32)
    b = torch.randn((8192, 2048), generator=g, dtype=torch.float32)
    return a.to(torch.bfloat16), b.t().contiguous().to(torch.bfloat16)


def ffn_up():
    """X [8192,8192] N(0,1); W [22016,8192] N(0,0.02^2) with an elementwise
    Bernoulli(0.001) outlier mask scaled x20; seed 3."""
    g = _gen(3)
    x = torch.randn((8192, 8192), generator=g, dtype=torch.float32).to(torch.bfloat16)
    w = torch.randn((22016, 8192), generator=g, dtype=torch.float32) * 0.02
    mask = torch.rand((22016, 8192), generator=g, dtype=torch.float32) < 0.001
    w[mask] *= 20.0
    return x, w.to(torch.bfloat16)


def decode():
    """Weights for the three linears (draw order up, down, qkv), each
    N(0,0.02^2) [N,K]; then X64 for K=4096 and X64 for K=14336, N(0,1).
    The M-token activation is the first M rows of X64.  Seed 4.
    Returns ({name: W}, {K: X64})."""
    g = _gen(4)
    ws = {}
    for name in ("up", "down", "qkv"):
        n, k = DECODE_SHAPES[name]
        ws[name] = randn_bf16((n, k), g, 0.02)
    xs = {4096: randn_bf16((64, 4096), g), 14336: randn_bf16((64, 14336), g)}
    return ws, xs


def random_bf16(shape, seed: int, sigma: float = 1.0) -> torch.Tensor:
    """Plain N(0, sigma^2) bf16 tensor for edge-case tests."""
    return randn_bf16(shape, _gen(seed), sigma)


def bits(t: torch.Tensor):
    """uint16 numpy view of a CPU bf16 tensor (what the oracle reads)."""
    import numpy as np
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
