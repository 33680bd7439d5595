"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module holds random-number generation only: no quantisation, no GEMM, none of
the method's arithmetic.  Shapes and distributions follow the workloads on the pages
(Qwen3.8-27B FFN matrices: gate/up [17408, 5120], down [5120, 17408]; weights
~ N(0, 0.02); activations ~ N(0, 1) rounded to bf16).

Seed convention: weights seed 0, activations seed 1, a second matrix seed 2, a third
seed 3, row samples seed 0.  Copies of a matrix in a weight ring use seed + 1000*i.
"""
from __future__ import annotations

import numpy as np
import torch

W_SEED, X_SEED, W2_SEED, W3_SEED, ROW_SEED = 0, 1, 2, 3, 0

# 27B FFN dimensions (Atlas issue, prefill kernel ranking: 2*3*5120*17408*7235*64).
HIDDEN = 5120
INTERMEDIATE = 17408


def weights(N: int, K: int, seed: int = W_SEED, std: float = 0.02) -> torch.Tensor:
    """float32 [N, K] ~ N(0, std^2), CPU, from torch's seeded generator."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(N, K, generator=g, dtype=torch.float32) * std


def activations(B: int, K: int, seed: int = X_SEED) -> torch.Tensor:
    """bf16 [B, K] ~ N(0, 1) (float32 draw, RNE to bf16), CPU."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(B, K, generator=g, dtype=torch.float32).to(torch.bfloat16)


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """uint16 view of a bf16 tensor's bit patterns (no arithmetic)."""
    assert x.dtype == torch.bfloat16
    return x.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bits_to_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def sample_rows(M: int, n: int = 62, seed: int = ROW_SEED) -> np.ndarray:
    """Sorted row indices: a seeded random subset of size n plus rows 0 and M-1."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    idx = torch.randperm(M, generator=g)[: min(n, M)].tolist()
    return np.array(sorted(set(idx) | {0, M - 1}), dtype=np.int64)


def one_hot(B: int, K: int, cols) -> torch.Tensor:
    """bf16 [B, K] with x[b, cols[b]] = 1 and zeros elsewhere."""
    x = torch.zeros(B, K, dtype=torch.bfloat16)
    for b, c in enumerate(cols):
        x[b, int(c)] = 1.0
    return x


def routing(T: int, E: int, k: int, seed: int = ROW_SEED):
    """Top-k routing of T tokens over E experts drawn at random (distinct experts per token).
    Returns (token index of each routed row, expert of each row, offsets int32 [E+1]) with the
    rows grouped by expert, tokens ascending within an expert."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    choice = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)])  # [T, k]
    tok = torch.arange(T).repeat_interleave(k)
    exp = choice.reshape(-1)
    order = torch.argsort(exp * T + tok)
    tok, exp = tok[order], exp[order]
    counts = torch.bincount(exp, minlength=E)
    off = torch.zeros(E + 1, dtype=torch.int32)
    off[1:] = torch.cumsum(counts, 0).to(torch.int32)
    return tok.numpy(), exp.numpy(), off.numpy()
