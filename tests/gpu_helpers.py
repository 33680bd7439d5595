"""Shared helpers for the GPU tests: upload oracle-packed weights, run the library through the
C ABI (via the thin binding), and compare with the oracle.

Every oracle input and expected value here comes from the seeded generators and ``oracle/``;
the CUDA path only produces the values under test."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from block_quantized_weight_qgemm_b200 import inputs
from block_quantized_weight_qgemm_b200 import qgemm

TOL = 1e-3  # max |y - y_ref| / (||x_b|| ||w_n||), the acceptance bound of the method


def upload_packed(fmt, codes: np.ndarray, scales: np.ndarray, ts: float, N: int, K: int):
    pw = qgemm.PackedWeight(fmt, N, K)
    pw.codes.copy_(torch.from_numpy(codes))
    pw.scales.copy_(torch.from_numpy(scales))
    if pw.tensor_scale is not None:
        pw.tensor_scale.fill_(ts)
    return pw


class Case:
    """One weight matrix: fp32 source, oracle packing, dequantised fp64 rows, device copy."""

    def __init__(self, fmt, N, K, seed=inputs.W_SEED, W=None):
        self.fmt, self.N, self.K = fmt, N, K
        self.W = inputs.weights(N, K, seed=seed).numpy() if W is None else W
        self.codes, self.scales, self.ts = oracle.pack(fmt, self.W)
        self.Wd = oracle.dequant(fmt, self.codes, self.scales, self.ts, N, K)
        self.pw = upload_packed(fmt, self.codes, self.scales, self.ts, N, K)


def x_bits(x_bf16: torch.Tensor) -> np.ndarray:
    return inputs.bf16_bits(x_bf16.cpu())


def gpu_run(case: Case, x_bf16: torch.Tensor, y_dtype=torch.float32) -> np.ndarray:
    x = x_bf16.cuda().contiguous()
    y = qgemm.run(x, case.pw, y_dtype=y_dtype)
    torch.cuda.synchronize()
    return y.float().cpu().numpy().astype(np.float64)


def norm_err(y_gpu, y_ref, xb, Wd) -> float:
    return oracle.normalised_error(y_gpu, y_ref, xb, Wd)


def silu(g):
    return g / (1.0 + np.exp(-g))


def dsilu(g):
    s = 1.0 / (1.0 + np.exp(-g))
    return s * (1.0 + g * (1.0 - s))


def h_bound_violations(h_gpu_bits, g, u, xb, Wg, Wu, tol=TOL):
    """FFN h check: |h - h_ref| <= 2^-8 |h_ref| + tol (|SiLU'(g) u| ||x|| ||wg|| +
    |SiLU(g)| ||x|| ||wu||): one bf16 ulp plus first-order propagation of the GEMM bound."""
    xd = oracle.bf16_decode_array(xb)
    xn = np.sqrt((xd * xd).sum(axis=1))[:, None]
    gn = np.sqrt((Wg * Wg).sum(axis=1))[None, :]
    un = np.sqrt((Wu * Wu).sum(axis=1))[None, :]
    h_ref = silu(g) * u
    h_gpu = oracle.bf16_decode_array(h_gpu_bits)
    bound = 2.0 ** -8 * np.abs(h_ref) + tol * (np.abs(dsilu(g) * u) * xn * gn + np.abs(silu(g)) * xn * un)
    bad = np.abs(h_gpu - h_ref) > bound
    return int(bad.sum()), float(np.max(np.abs(h_gpu - h_ref) / np.maximum(bound, 1e-300)))


def bf16_bits_of(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def round_f16(a: np.ndarray) -> np.ndarray:
    return a.astype(np.float16).astype(np.float64)


def round_bf16(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()
