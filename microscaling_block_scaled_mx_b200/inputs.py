"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no MX arithmetic: it only draws random tensors (numpy PCG64)
and rounds float32 to bf16 where a workload is stated in bf16.  Both the CUDA
path (through the binding) and the CPU oracle (in the tests and the benchmark's
CPU baseline) consume exactly the bytes produced here.

Workloads (sizes and distributions; the pages train on datasets and models
that are not available, so these stand in for them):
  * round trip + GEMM: fp32 A 256x512, B 512x256, N(0,1) x 2^U per row with
    U ~ Uniform(-8, 8), 1% exact zeros, 0.1% fp32 subnormals.
  * cast bandwidth sweep: bf16 8192x8192 N(0,1), 0.01% of positions x 1e3.
  * GPT-2-small-shaped MXFP8 GEMMs: activations N(0,1) M=8192 x K (768, 3072),
    weights N(0, 0.02^2) stored N x K (3072x768, 768x3072), bf16.
  * Llama-3-8B-shaped MXFP4 GEMMs: activations 8192 x (4096, 14336) N(0,1),
    weights (6144x4096, 14336x4096, 4096x14336) N(0, 0.02^2), bf16.
  * weight gradient: dY 16384x4096 and X 16384x14336 bf16, Student-t nu=3.
"""
from __future__ import annotations

import numpy as np

SEED_BASE = 1000


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 (round to nearest even, via torch's CPU cast), as uint16 bits."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def rng_for(config_index: int, stream: int = 0) -> np.random.Generator:
    return np.random.default_rng([SEED_BASE + config_index, stream])


def _subnormals(rng, n):
    sign = rng.integers(0, 2, n, dtype=np.uint32) << 31
    mant = rng.integers(1, 1 << 23, n, dtype=np.uint32)
    return (sign | mant).view(np.float32)


def roundtrip_matrix(rows: int, cols: int, rng: np.random.Generator) -> np.ndarray:
    """N(0,1) x 2^U per row, 1% exact zeros, 0.1% fp32 subnormals (float32)."""
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    x *= np.exp2(rng.uniform(-8.0, 8.0, (rows, 1))).astype(np.float32)
    n = rows * cols
    flat = x.reshape(-1)
    flat[rng.choice(n, size=n // 100, replace=False)] = 0.0
    k = n // 1000
    flat[rng.choice(n, size=k, replace=False)] = _subnormals(rng, k)
    return x


def config_roundtrip():
    rng = rng_for(0)
    return {"A": roundtrip_matrix(256, 512, rng), "B": roundtrip_matrix(512, 256, rng)}


def cast_sweep_input(rows: int = 8192, cols: int = 8192, seed_stream: int = 0) -> np.ndarray:
    """bf16 bits: N(0,1) with 0.01% of positions multiplied by 1e3."""
    rng = rng_for(1, seed_stream)
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    n = rows * cols
    flat = x.reshape(-1)
    idx = rng.choice(n, size=max(1, n // 10000), replace=False)
    flat[idx] *= np.float32(1e3)
    return to_bf16_bits(x)


def linear_operands(M: int, K: int, N: int, config_index: int, stream: int = 0):
    """bf16 bits: activations X (M x K) ~ N(0,1), weight W (N x K) ~ N(0, 0.02^2)."""
    rng = rng_for(config_index, stream)
    x = rng.standard_normal((M, K), dtype=np.float32)
    w = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    return to_bf16_bits(x), to_bf16_bits(w)


GPT2_GEMMS = [(8192, 3072, 768), (8192, 768, 3072)]           # (M, N, K)
LLAMA3_GEMMS = [(8192, 6144, 4096), (8192, 14336, 4096), (8192, 4096, 14336)]
WGRAD_SHAPE = (16384, 4096, 14336)                             # tokens, d_out, d_in


def wgrad_operands(tokens: int = 16384, d_out: int = 4096, d_in: int = 14336):
    """bf16 bits: dY (tokens x d_out) and X (tokens x d_in), Student-t nu = 3."""
    rng = rng_for(4)
    dy = rng.standard_t(3, size=(tokens, d_out)).astype(np.float32)
    x = rng.standard_t(3, size=(tokens, d_in)).astype(np.float32)
    return to_bf16_bits(dy), to_bf16_bits(x)
