"""Seeded synthetic inputs for the NVFP4 decode GEMM.

This module draws random bytes and bf16 activations and nothing else: it holds
none of the method's arithmetic (no code decoding, no products, no sums), so
the CUDA path and the float64 oracle can both be fed from it.

Recipes (ignis, "Models and artifacts", "The artifact": a 4-bit floating point
body with one scale per 16 values; the distributions are the workload's):
  * element codes: every nibble independent and uniform over the 16 E2M1
    codes, i.e. every byte of the canonical code plane uniform over 0..255;
  * scale codes: sign 0, exponent e uniform over an inclusive integer range,
    mantissa uniform over 0..7, byte = ((e + 7) << 3) | mantissa;
  * X: N(0, 1) drawn in float64, rounded to float32, then to bf16 with
    round-to-nearest-even; the bf16 bit patterns are the ground truth.
Every tensor of every workload has its own stream:
``SeedSequence(seed, spawn_key=(workload_id, tensor_id))``.
"""
from __future__ import annotations

import numpy as np

# Scale exponent ranges of the workloads (inclusive).
EXP_UNIFORM_M4_2 = (-4, 2)   # "uniform over exponents 2^-4..2^2"
EXP_LOGU_M6_4 = (-6, 4)      # "log-uniform over 2^-6..2^4"
GSCALE = 1.0 / 64.0


def rng(workload_id: int, tensor_id: int, seed: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(
        np.random.SeedSequence(seed, spawn_key=(int(workload_id), int(tensor_id)))))


def codes(g: np.random.Generator, N: int, K: int) -> np.ndarray:
    """Canonical element plane u8[N][K/2], every nibble uniform."""
    assert K % 2 == 0
    return g.integers(0, 256, size=(N, K // 2), dtype=np.uint8)


def scales(g: np.random.Generator, N: int, K: int, exp_range=EXP_UNIFORM_M4_2) -> np.ndarray:
    """Canonical scale plane u8[N][K/16] of positive normal E4M3 codes."""
    assert K % 16 == 0
    lo, hi = exp_range
    e = g.integers(lo, hi + 1, size=(N, K // 16), dtype=np.int64)
    m = g.integers(0, 8, size=(N, K // 16), dtype=np.int64)
    return (((e + 7) << 3) | m).astype(np.uint8)


def bf16_bits_from_f64(a: np.ndarray) -> np.ndarray:
    """float64 -> float32 (RNE) -> bf16 (RNE); returns the uint16 bit patterns."""
    f = np.ascontiguousarray(a, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def activations(g: np.random.Generator, M: int, K: int) -> np.ndarray:
    """bf16 bit patterns of X[M][K] ~ N(0, 1)."""
    return bf16_bits_from_f64(g.standard_normal(size=(M, K)))


def matrix(workload_id: int, tensor_id: int, N: int, K: int, exp_range=EXP_UNIFORM_M4_2,
           seed: int = 0):
    """(codes, scales) of one N x K matrix from its own stream."""
    g = rng(workload_id, tensor_id, seed)
    return codes(g, N, K), scales(g, N, K, exp_range)


# The workloads: shapes and value recipes.
WORKLOADS = {
    0: dict(name="gemm_m1_n256_k512", N=256, K=512, M=(1,), exp=EXP_UNIFORM_M4_2),
    1: dict(name="proj_n5120_k5120", N=5120, K=5120, M=(1, 2, 4, 8), exp=EXP_UNIFORM_M4_2),
    2: dict(name="mlp_gateup2x17408_down5120_k5120", Nff=17408, K=5120, M=(1, 8),
            exp=EXP_UNIFORM_M4_2),
    3: dict(name="head_n151936_k5120", N=151936, K=5120, M=(1, 4, 8), exp=EXP_LOGU_M6_4),
    4: dict(name="round_64layers_head_m1to8", layers=64, hidden=5120, ffn=17408,
            vocab=151936, M=tuple(range(1, 9)), exp=EXP_UNIFORM_M4_2),
}


def torch_matrix(workload_id: int, tensor_id: int, N: int, K: int, device,
                 exp_range=EXP_UNIFORM_M4_2, seed: int = 0):
    """(codes, scales) drawn on a torch device (for multi-GB workloads).

    Same recipe as ``matrix`` with torch's generator for that device, seeded
    from the workload and tensor ids; draws are reproducible per device type.
    """
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed((int(seed) * 1000003 + int(workload_id) * 65537 + int(tensor_id)) & (2**63 - 1))
    q = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=device, generator=gen)
    lo, hi = exp_range
    e = torch.randint(lo + 7, hi + 8, (N, K // 16), dtype=torch.uint8, device=device, generator=gen)
    m = torch.randint(0, 8, (N, K // 16), dtype=torch.uint8, device=device, generator=gen)
    s = (e << 3) | m
    return q, s


def torch_activations(workload_id: int, tensor_id: int, M: int, K: int, device, seed: int = 0):
    """bf16 X[M][K] ~ N(0, 1) drawn on a torch device (float64 -> float32 -> bf16, RNE)."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed((int(seed) * 1000003 + int(workload_id) * 65537 + 7919 * (int(tensor_id) + 1))
                    & (2**63 - 1))
    return torch.randn((M, K), dtype=torch.float64, device=device, generator=gen) \
        .to(torch.float32).to(torch.bfloat16)
