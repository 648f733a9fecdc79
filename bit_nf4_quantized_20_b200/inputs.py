"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

Holds none of the layer's arithmetic: it only draws normal samples with torch's
generator and rounds them to BF16.  Both the GPU path and the CPU oracle take
their inputs from here (the oracle receives copies of the same bytes).

Seed recipe: seed = 1_000_000 * config + 1_000 * layer + 10 * proj + tensor,
tensor in {W: 0, X: 1, A: 2, B: 3, dY: 4}.

Distributions (the workloads the layer is measured on): W ~ N(0, 0.02^2),
X ~ N(0, 1), A ~ N(0, 1/K), B ~ N(0, 0.01^2), dY ~ N(0, 1).
"""
from __future__ import annotations

import math

import torch

TENSOR_ID = {"W": 0, "X": 1, "A": 2, "B": 3, "dY": 4}

# Llama-3.1-8B block: (name, N_out, K_in)
LLAMA8B_PROJ = [("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096), ("o", 4096, 4096),
                ("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336)]
# 65B-shaped block (hidden 8192, ffn 22016, 64-head MHA)
LLAMA65B_PROJ = [("q", 8192, 8192), ("k", 8192, 8192), ("v", 8192, 8192), ("o", 8192, 8192),
                 ("gate", 22016, 8192), ("up", 22016, 8192), ("down", 8192, 22016)]


def seed_of(config: int, layer: int, proj: int, tensor: str) -> int:
    return 1_000_000 * config + 1_000 * layer + 10 * proj + TENSOR_ID[tensor]


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """std * N(0, 1) drawn in fp32 with a seeded generator, rounded to BF16."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    x = torch.randn(tuple(shape), generator=g, device=dev, dtype=torch.float32)
    return (x * float(std)).to(torch.bfloat16)


def layer_inputs(config: int, layer: int, proj: int, T: int, N: int, K: int, r: int,
                 device="cpu", a_std: float | None = None, b_std: float = 0.01):
    """W[N, K], X[T, K], A[r, K], B[N, r], dY[T, N] as BF16 tensors."""
    a_std = math.sqrt(1.0 / K) if a_std is None else a_std
    W = normal_bf16((N, K), 0.02, seed_of(config, layer, proj, "W"), device)
    X = normal_bf16((T, K), 1.0, seed_of(config, layer, proj, "X"), device)
    A = normal_bf16((r, K), a_std, seed_of(config, layer, proj, "A"), device)
    B = normal_bf16((N, r), b_std, seed_of(config, layer, proj, "B"), device)
    dY = normal_bf16((T, N), 1.0, seed_of(config, layer, proj, "dY"), device)
    return W, X, A, B, dY


def bf16_bits(t: torch.Tensor):
    """uint16 NumPy view of a BF16 tensor's bit patterns (copied to host)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
