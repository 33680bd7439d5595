"""CPU oracle for the block-quantized-weight GEMM -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import this module.  The CUDA library never uses it.

This is a thin ctypes shim over ``qgemm_oracle.c`` (plain C, fp64): argument
marshalling only, every number is computed in the C file.  The shared library is
compiled with gcc on first use (``build()``), in-tree, next to the source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

Q8_0, NVFP4, MXFP4, FP8 = 0, 1, 2, 3
FORMATS = {"q8_0": Q8_0, "nvfp4": NVFP4, "mxfp4": MXFP4, "fp8": FP8}

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qgemm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math: IEEE semantics are the point)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
             "-pthread", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            d, u, i64, vp = ctypes.c_double, ctypes.c_uint, ctypes.c_int64, ctypes.c_void_p
            for name in ("orc_e2m1", "orc_e4m3", "orc_e8m0", "orc_f16", "orc_bf16"):
                getattr(lib, name).restype = d
                getattr(lib, name).argtypes = [u]
            lib.orc_e2m1_encode.restype = u
            lib.orc_e2m1_encode.argtypes = [d]
            lib.orc_e4m3_encode_pos.restype = u
            lib.orc_e4m3_encode_pos.argtypes = [d]
            lib.orc_e4m3_encode.restype = u
            lib.orc_e4m3_encode.argtypes = [d]
            lib.orc_f16_encode_satfinite.restype = u
            lib.orc_f16_encode_satfinite.argtypes = [d]
            lib.orc_bf16_encode.restype = u
            lib.orc_bf16_encode.argtypes = [d]
            lib.orc_silu.restype = d
            lib.orc_silu.argtypes = [d]
            lib.orc_code_pitch.restype = i64
            lib.orc_code_pitch.argtypes = [ctypes.c_int, i64]
            lib.orc_scale_pitch.restype = i64
            lib.orc_scale_pitch.argtypes = [ctypes.c_int, i64]
            lib.orc_pack_q8_0.argtypes = [vp, i64, i64, vp, vp]
            lib.orc_pack_nvfp4.argtypes = [vp, i64, i64, vp, vp, vp]
            lib.orc_pack_mxfp4.argtypes = [vp, i64, i64, vp, vp]
            lib.orc_pack_fp8.argtypes = [vp, i64, i64, vp, vp]
            lib.orc_split_x.argtypes = [vp, i64, i64, ctypes.c_int, ctypes.c_int, vp]
            lib.orc_split_x_bs.argtypes = [vp, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, vp]
            lib.orc_dequant.argtypes = [ctypes.c_int, vp, vp, ctypes.c_float, i64, i64, vp]
            lib.orc_gemm.argtypes = [vp, i64, i64, vp, i64, vp, ctypes.c_int]
            lib.orc_ffn_gate_up.argtypes = [vp, i64, i64, vp, vp, i64, vp, vp, vp, ctypes.c_int]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _fmt(fmt) -> int:
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# ---- scalar decoders / encoders ---------------------------------------------------------

def e2m1(code: int) -> float:
    return _load().orc_e2m1(code)


def e4m3(byte: int) -> float:
    return _load().orc_e4m3(byte)


def e8m0(byte: int) -> float:
    return _load().orc_e8m0(byte)


def f16(bits: int) -> float:
    return _load().orc_f16(bits)


def bf16(bits: int) -> float:
    return _load().orc_bf16(bits)


def e2m1_encode(v: float) -> int:
    return _load().orc_e2m1_encode(v)


def e4m3_encode_pos(v: float) -> int:
    return _load().orc_e4m3_encode_pos(v)


def e4m3_encode(v: float) -> int:
    return _load().orc_e4m3_encode(v)


def f16_encode_satfinite(v: float) -> int:
    return _load().orc_f16_encode_satfinite(v)


def bf16_encode(v: float) -> int:
    return _load().orc_bf16_encode(v)


def silu(g: float) -> float:
    return _load().orc_silu(g)


# ---- layout -----------------------------------------------------------------------------

def block_size(fmt) -> int:
    return 16 if _fmt(fmt) in (NVFP4, FP8) else 32


def code_pitch(fmt, K: int) -> int:
    return int(_load().orc_code_pitch(_fmt(fmt), K))


def scale_pitch(fmt, K: int) -> int:
    return int(_load().orc_scale_pitch(_fmt(fmt), K))


# ---- array routines ---------------------------------------------------------------------

def pack(fmt, W: np.ndarray):
    """W: float32 [N, K].  Returns (codes uint8 [N, cpitch], scales uint8 [N, spitch], ts).
    FP8 has no block scales (spitch = 0); NVFP4 and FP8 return their fp32 tensor scale, the
    other formats 1.0."""
    f = _fmt(fmt)
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    codes = np.zeros((N, code_pitch(f, K)), dtype=np.uint8)
    scales = np.zeros((N, scale_pitch(f, K)), dtype=np.uint8)
    ts = np.zeros(1, dtype=np.float32)
    lib = _load()
    if f == Q8_0:
        lib.orc_pack_q8_0(_ptr(W), N, K, _ptr(codes), _ptr(scales))
        tsv = 1.0
    elif f == NVFP4:
        lib.orc_pack_nvfp4(_ptr(W), N, K, _ptr(codes), _ptr(scales), _ptr(ts))
        tsv = float(ts[0])
    elif f == FP8:
        lib.orc_pack_fp8(_ptr(W), N, K, _ptr(codes), _ptr(ts))
        tsv = float(ts[0])
    else:
        lib.orc_pack_mxfp4(_ptr(W), N, K, _ptr(codes), _ptr(scales))
        tsv = 1.0
    return codes, scales, tsv


def dequant(fmt, codes: np.ndarray, scales: np.ndarray, ts: float, N: int, K: int) -> np.ndarray:
    f = _fmt(fmt)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    assert codes.shape == (N, code_pitch(f, K)) and scales.shape == (N, scale_pitch(f, K))
    Wd = np.zeros((N, K), dtype=np.float64)
    _load().orc_dequant(f, _ptr(codes), _ptr(scales), ctypes.c_float(ts), N, K, _ptr(Wd))
    return Wd


def gemm(x16: np.ndarray, Wd: np.ndarray, nthreads: int | None = None) -> np.ndarray:
    """x16: uint16 bf16 bit patterns [B, K]; Wd: float64 [N, K] -> y float64 [B, N]."""
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    Wd = np.ascontiguousarray(Wd, dtype=np.float64)
    B, K = x16.shape
    N, K2 = Wd.shape
    assert K == K2
    y = np.zeros((B, N), dtype=np.float64)
    _load().orc_gemm(_ptr(x16), B, K, _ptr(Wd), N, _ptr(y), nthreads or default_threads())
    return y


def split_x(x16: np.ndarray, elem: str, terms: int) -> np.ndarray:
    """x (bf16 bits [B, K]) peeled into `terms` E4M3 ("e4m3") or E2M1 ("e2m1") terms per
    32-block, each with its own power-of-two scale; returns the sum of the terms (fp64)."""
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    B, K = x16.shape
    xs = np.zeros((B, K), dtype=np.float64)
    _load().orc_split_x(_ptr(x16), B, K, 0 if elem == "e4m3" else 1, terms, _ptr(xs))
    return xs


# block size, prescale shift, smallest scale exponent, term element (0 E4M3, 1 E2M1) and
# number of terms of the block-scaled path's split, per weight format
BS_SPLIT = {"mxfp4": (32, 0, -127, 1, 3), "nvfp4": (16, 10, -9, 1, 3), "fp8": (32, 0, -127, 0, 2)}


def split_x_bs(x16: np.ndarray, fmt: str, terms: int | None = None) -> np.ndarray:
    """The activation split as the block-scaled path of weight format `fmt` applies it: per-row
    power-of-two prescale, E2M1 (FP4 weights) or E4M3 (FP8 weights) terms with power-of-two
    block scales in the MMA scale type's range (orc_split_x_bs); returns 2^xe * the sum of the
    terms (fp64).  terms defaults to the path's own (3 E2M1, 2 E4M3)."""
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    B, K = x16.shape
    blk, xshift, emin, elem, nterms = BS_SPLIT[fmt]
    xs = np.zeros((B, K), dtype=np.float64)
    _load().orc_split_x_bs(_ptr(x16), B, K, blk, xshift, emin, elem,
                           nterms if terms is None else terms, _ptr(xs))
    return xs


def gemm_f64(xd: np.ndarray, Wd: np.ndarray) -> np.ndarray:
    """y = xd Wd^T for an fp64 x (the split activations) -- numpy's fp64 matmul."""
    return np.asarray(xd, dtype=np.float64) @ np.asarray(Wd, dtype=np.float64).T


def ffn_gate_up(x16: np.ndarray, Wg: np.ndarray, Wu: np.ndarray, nthreads: int | None = None):
    """Returns (g, u, h16): g, u float64 [M, N]; h16 uint16 bf16 bits of SiLU(g)*u."""
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    Wg = np.ascontiguousarray(Wg, dtype=np.float64)
    Wu = np.ascontiguousarray(Wu, dtype=np.float64)
    M, K = x16.shape
    N = Wg.shape[0]
    assert Wg.shape == (N, K) and Wu.shape == (N, K)
    g = np.zeros((M, N), dtype=np.float64)
    u = np.zeros((M, N), dtype=np.float64)
    h = np.zeros((M, N), dtype=np.uint16)
    _load().orc_ffn_gate_up(_ptr(x16), M, K, _ptr(Wg), _ptr(Wu), N, _ptr(g), _ptr(u), _ptr(h),
                            nthreads or default_threads())
    return g, u, h


def normalised_error(y_test: np.ndarray, y_ref: np.ndarray, x16: np.ndarray, Wd: np.ndarray) -> float:
    """max_{b,n} |y_test - y_ref| / (||x_b||_2 * ||w_n||_2), w_n the dequantised row.

    Rows or columns with a zero norm are compared absolutely (the denominator is
    replaced by 1): their exact result is 0."""
    xd = np.vectorize(bf16, otypes=[np.float64])(x16) if x16.size < 4096 else _bf16_array(x16)
    xn = np.sqrt((xd * xd).sum(axis=1))
    wn = np.sqrt((Wd * Wd).sum(axis=1))
    den = np.outer(xn, wn)
    den[den == 0] = 1.0
    return float(np.max(np.abs(np.asarray(y_test, dtype=np.float64) - y_ref) / den))


def _bf16_array(x16: np.ndarray) -> np.ndarray:
    """Decode a bf16 bit array through the oracle's decoder, via a 65536-entry table."""
    table = bf16_table()
    return table[np.asarray(x16, dtype=np.uint16).astype(np.int64)]


_bf16_tab = None


def bf16_table() -> np.ndarray:
    global _bf16_tab
    if _bf16_tab is None:
        lib = _load()
        _bf16_tab = np.array([lib.orc_bf16(i) for i in range(65536)], dtype=np.float64)
    return _bf16_tab


def bf16_decode_array(x16: np.ndarray) -> np.ndarray:
    return _bf16_array(x16)
