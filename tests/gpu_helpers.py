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


def tile_packed(fmt, codes_rm: np.ndarray, scales_rm: np.ndarray, N: int, K: int):
    """The tile-major layout of include/qgemm.h, built from the row-major packing with numpy
    (a byte permutation written from the header's description, independent of the library)."""
    f = oracle.FORMATS[fmt] if isinstance(fmt, str) else fmt
    byte_codes = f in (oracle.Q8_0, oracle.FP8)
    CK = 128 if byte_codes else 256
    SB = {oracle.Q8_0: 8, oracle.NVFP4: 16, oracle.MXFP4: 8, oracle.FP8: 0}[f]
    T, C = -(-N // 128), -(-K // CK)
    row_code = K if byte_codes else K // 2
    row_scale = {oracle.Q8_0: 2 * (K // 32), oracle.NVFP4: K // 16, oracle.MXFP4: K // 32,
                 oracle.FP8: 0}[f]
    cfull = np.zeros((T * 128, C * 128), dtype=np.uint8)
    cfull[:N, :row_code] = codes_rm[:, :row_code]
    grp = cfull.reshape(T, 128, C, 8, 16).transpose(0, 2, 1, 3, 4)  # [T][C][row][group][16]
    out = np.empty_like(grp)
    for r in range(128):
        perm = [g ^ (r & 7) for g in range(8)]
        out[:, :, r, perm, :] = grp[:, :, r, :, :]
    sfull = np.zeros((T * 128, C * SB), dtype=np.uint8)
    sfull[:N, :row_scale] = scales_rm[:, :row_scale]
    st = sfull.reshape(T, 128, C, SB).transpose(0, 2, 1, 3)
    return np.ascontiguousarray(out).reshape(-1), np.ascontiguousarray(st).reshape(-1)


def upload_packed(fmt, codes: np.ndarray, scales: np.ndarray, ts: float, N: int, K: int):
    """Oracle row-major packing -> tile-major device buffers (numpy permutation + copy)."""
    pw = qgemm.PackedWeight(fmt, N, K)
    ct, st = tile_packed(fmt, codes, scales, N, K)
    pw.codes.copy_(torch.from_numpy(ct))
    pw.scales.copy_(torch.from_numpy(st))
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
