"""Thin ctypes binding of libqgemm.so (the C ABI in include/qgemm.h).

Argument marshalling only: every step of the computation runs in the CUDA library.  The
functions mirror the C names; torch tensors stand in for device pointers and torch's
current stream is passed as `stream`.  The library is loaded on first use; if it is
missing or fails to load, the call raises -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

Q8_0, NVFP4, MXFP4, FP8 = 0, 1, 2, 3
FORMATS = {"q8_0": Q8_0, "nvfp4": NVFP4, "mxfp4": MXFP4, "fp8": FP8}
Y_F32, Y_BF16 = 0, 1
BLOCK = {Q8_0: 32, NVFP4: 16, MXFP4: 32, FP8: 16}  # K granularity (FP8: no block scales)
TENSOR_SCALE = (NVFP4, FP8)

OK = 0
STATUS = {
    0: "QGEMM_OK", 1: "QGEMM_ERR_FORMAT", 2: "QGEMM_ERR_SHAPE", 3: "QGEMM_ERR_K_BLOCK",
    4: "QGEMM_ERR_NULL", 5: "QGEMM_ERR_ALIGN", 6: "QGEMM_ERR_WORKSPACE", 7: "QGEMM_ERR_CUDA",
    8: "QGEMM_ERR_DEVICE", 9: "QGEMM_ERR_DEVICE_TIMEOUT", 10: "QGEMM_ERR_DEVICE_ARG",
}

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqgemm.so")
_lib = None
_lock = threading.Lock()

# (name, restype, argtypes) of every exported entry point
_I64, _SZ, _VP, _I = ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int
SIGNATURES = [
    ("qgemm_packed_size", _I, [_I, _I64, _I64, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)]),
    ("qgemm_packed_geometry", _I, [_I, _I64, _I64, ctypes.POINTER(_I64), ctypes.POINTER(_I64),
                                   ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    ("qgemm_row_pitches", _I, [_I, _I64, ctypes.POINTER(_I64), ctypes.POINTER(_I64)]),
    ("qgemm_repack_rowmajor", _I, [_I, _I64, _I64, _VP, _I64, _VP, _I64, _VP, _VP, _VP]),
    ("qgemm_pack", _I, [_I, _VP, _I64, _I64, _VP, _VP, _VP, _VP]),
    ("qgemm_workspace_size", _I, [_I, _I64, _I64, _I64, ctypes.POINTER(_SZ)]),
    ("qgemm_run", _I, [_I, _VP, _I64, _I64, _VP, _VP, _VP, _I64, _VP, _I, _VP, _SZ, _VP]),
    ("qgemm_run_noalloc", _I, [_I, _VP, _I64, _I64, _VP, _VP, _VP, _I64, _VP, _I, _VP]),
    ("qgemm_ffn_workspace_size", _I, [_I, _I64, _I64, _I64, ctypes.POINTER(_SZ)]),
    ("qgemm_ffn_gate_up", _I, [_I, _VP, _I64, _I64, _VP, _VP, _VP, _VP, _VP, _VP, _I64, _VP, _VP,
                               _SZ, _VP]),
    ("qgemm_moe_workspace_size", _I, [_I, _I64, _I64, _I64, _I64, ctypes.POINTER(_SZ)]),
    ("qgemm_moe_run", _I, [_I, _VP, _I64, _I64, _I, _VP, _I64, _VP, _VP, _VP, _I64, _VP, _I, _VP,
                           _SZ, _VP]),
    ("qgemm_moe_gate_up", _I, [_I, _VP, _I64, _I64, _I, _VP, _I64, _VP, _VP, _VP, _VP, _VP, _VP,
                               _I64, _VP, _VP, _SZ, _VP]),
    ("qgemm_bs_split_size", _I, [_I, _I64, _I64, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ),
                                 ctypes.POINTER(_SZ)]),
    ("qgemm_bs_split_x", _I, [_I, _VP, _I64, _I64, _VP, _VP, _VP, _VP]),
    ("qgemm_bs_workspace_size", _I, [_I, _I64, _I64, _I64, ctypes.POINTER(_SZ)]),
    ("qgemm_bs_run", _I, [_I, _VP, _I64, _I64, _VP, _VP, _VP, _I64, _VP, _I, _VP, _SZ, _VP]),
    ("qgemm_bs_ffn_workspace_size", _I, [_I, _I64, _I64, _I64, ctypes.POINTER(_SZ)]),
    ("qgemm_bs_ffn_gate_up", _I, [_I, _VP, _I64, _I64, _VP, _VP, _VP, _VP, _VP, _VP, _I64, _VP,
                                  _VP, _SZ, _VP]),
    ("qgemm_split_k", _I, [_I, _I64, _I64, ctypes.POINTER(_I)]),
    ("qgemm_device_status", _I, [_I]),
    ("qgemm_profile_events", _I, [_VP, _VP]),
    ("qgemm_status_str", ctypes.c_char_p, [_I]),
    ("qgemm_last_cuda_error", ctypes.c_char_p, []),
]


class QgemmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        lib = _lib
        detail = lib.qgemm_status_str(status).decode() if lib else ""
        cuda = lib.qgemm_last_cuda_error().decode() if (lib and status == 7) else ""
        super().__init__("%s: %s (%s)%s" % (where, STATUS.get(status, status), detail,
                                            (" -- " + cuda) if cuda else ""))


def lib():
    """The loaded library (raises if libqgemm.so is missing: build it first)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError("libqgemm.so not found at %s; run "
                                   "`python -m block_quantized_weight_qgemm_b200.build`" % LIB_PATH)
            handle = ctypes.CDLL(LIB_PATH)
            for name, res, args in SIGNATURES:
                fn = getattr(handle, name)
                fn.restype = res
                fn.argtypes = args
            _lib = handle
    return _lib


def _fmt(fmt) -> int:
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


def _check(status: int, where: str):
    if status != OK:
        raise QgemmError(status, where)


def _ptr(t):
    """Device address of a tensor (None for a missing or empty one)."""
    return None if (t is None or t.numel() == 0) else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ---- sizes -----------------------------------------------------------------------------

def packed_size(fmt, N: int, K: int):
    cb, sb = _SZ(), _SZ()
    _check(lib().qgemm_packed_size(_fmt(fmt), N, K, ctypes.byref(cb), ctypes.byref(sb)),
           "qgemm_packed_size")
    return cb.value, sb.value


def packed_geometry(fmt, N: int, K: int):
    """(row tiles T, chunks C, elements per chunk CK, scale bytes per row per chunk SB)."""
    t, c, ck, sb = _I64(), _I64(), _I(), _I()
    _check(lib().qgemm_packed_geometry(_fmt(fmt), N, K, ctypes.byref(t), ctypes.byref(c),
                                       ctypes.byref(ck), ctypes.byref(sb)), "qgemm_packed_geometry")
    return t.value, c.value, ck.value, sb.value


def row_pitches(fmt, K: int):
    cp, sp = _I64(), _I64()
    _check(lib().qgemm_row_pitches(_fmt(fmt), K, ctypes.byref(cp), ctypes.byref(sp)),
           "qgemm_row_pitches")
    return cp.value, sp.value


def workspace_size(fmt, N: int, K: int, B: int) -> int:
    b = _SZ()
    _check(lib().qgemm_workspace_size(_fmt(fmt), N, K, B, ctypes.byref(b)), "qgemm_workspace_size")
    return b.value


def ffn_workspace_size(fmt, N: int, K: int, M: int) -> int:
    b = _SZ()
    _check(lib().qgemm_ffn_workspace_size(_fmt(fmt), N, K, M, ctypes.byref(b)),
           "qgemm_ffn_workspace_size")
    return b.value


def split_k(fmt, N: int, K: int) -> int:
    s = _I()
    _check(lib().qgemm_split_k(_fmt(fmt), N, K, ctypes.byref(s)), "qgemm_split_k")
    return s.value


def device_status(reset: bool = True) -> int:
    return lib().qgemm_device_status(1 if reset else 0)


def profile_events(begin=None, end=None):
    """Record torch.cuda.Event `begin` / `end` around the next GEMM kernel launches."""
    lib().qgemm_profile_events(ctypes.c_void_p(begin.cuda_event) if begin is not None else None,
                               ctypes.c_void_p(end.cuda_event) if end is not None else None)


# ---- packed weights ---------------------------------------------------------------------

class PackedWeight:
    """Device buffers of one packed [N, K] matrix (codes, block scales -- empty for FP8 --
    and the fp32 tensor scale of NVFP4 and FP8)."""

    def __init__(self, fmt, N: int, K: int, device=None):
        self.fmt = _fmt(fmt)
        self.N, self.K = N, K
        device = device or torch.device("cuda", torch.cuda.current_device())
        cb, sb = packed_size(self.fmt, N, K)
        self.codes = torch.empty(cb, dtype=torch.uint8, device=device)   # tile-major layout
        self.scales = torch.empty(sb, dtype=torch.uint8, device=device)
        self.tensor_scale = (torch.empty(1, dtype=torch.float32, device=device)
                             if self.fmt in TENSOR_SCALE else None)

    @property
    def nbytes(self) -> int:
        """Algorithmic bytes a GEMM reads for this matrix (codes + scales, no row padding)."""
        code = self.N * (self.K if self.fmt in (Q8_0, FP8) else self.K // 2)
        if self.fmt == FP8:
            scale = 0
        else:
            scale = self.N * (2 * self.K // 32 if self.fmt == Q8_0 else self.K // BLOCK[self.fmt])
        return code + scale


def pack(fmt, W: torch.Tensor, stream=None, out: PackedWeight | None = None) -> PackedWeight:
    """qgemm_pack: W fp32 [N, K] on the device -> PackedWeight."""
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous()
    N, K = W.shape
    pw = out or PackedWeight(fmt, N, K, W.device)
    _check(lib().qgemm_pack(pw.fmt, _ptr(W), N, K, _ptr(pw.codes), _ptr(pw.scales),
                            _ptr(pw.tensor_scale), None, _stream(stream)), "qgemm_pack")
    return pw


def repack_rowmajor(fmt, codes_rm: torch.Tensor, scales_rm: torch.Tensor, N: int, K: int,
                    stream=None, out: PackedWeight | None = None) -> PackedWeight:
    """qgemm_repack_rowmajor: row-major interchange layout [N, pitch] -> PackedWeight."""
    assert codes_rm.is_cuda and scales_rm.is_cuda and codes_rm.dim() == 2 and scales_rm.dim() == 2
    pw = out or PackedWeight(fmt, N, K, codes_rm.device)
    spitch = scales_rm.stride(0) if scales_rm.numel() else 0
    _check(lib().qgemm_repack_rowmajor(pw.fmt, N, K, _ptr(codes_rm), codes_rm.stride(0),
                                       _ptr(scales_rm), spitch, _ptr(pw.codes),
                                       _ptr(pw.scales), _stream(stream)), "qgemm_repack_rowmajor")
    return pw


def run(x: torch.Tensor, pw: PackedWeight, y: torch.Tensor | None = None, y_dtype=torch.float32,
        workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """qgemm_run: x bf16 [B, K] (device) -> y [B, N] (fp32 or bf16)."""
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2
    B, K = x.shape
    assert K == pw.K
    if y is None:
        y = torch.empty((B, pw.N), dtype=y_dtype, device=x.device)
    ydt = Y_BF16 if y.dtype == torch.bfloat16 else Y_F32
    if workspace is None:
        nbytes = workspace_size(pw.fmt, pw.N, K, B)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    _check(lib().qgemm_run(pw.fmt, _ptr(x), B, K, _ptr(pw.codes), _ptr(pw.scales),
                           _ptr(pw.tensor_scale), pw.N, _ptr(y), ydt, _ptr(workspace),
                           workspace.numel(), _stream(stream)), "qgemm_run")
    return y


def bs_split_size(fmt, M: int, K: int) -> tuple[int, int, int]:
    """qgemm_bs_split_size: (code bytes, scale bytes, exponent bytes) of the split of x for
    weight format fmt (MXFP4, NVFP4 or FP8)."""
    c, sc, e = _SZ(), _SZ(), _SZ()
    _check(lib().qgemm_bs_split_size(_fmt(fmt), M, K, ctypes.byref(c), ctypes.byref(sc),
                                     ctypes.byref(e)), "qgemm_bs_split_size")
    return c.value, sc.value, e.value


def bs_split_x(x: torch.Tensor, fmt="mxfp4", stream=None):
    """qgemm_bs_split_x: x bf16 [M, K] -> (codes u8, scales u8, x_exp int32) in the layout of
    include/qgemm.h (three E2M1 terms per row for MXFP4 / NVFP4, two E4M3 terms for FP8, with the
    MMA's block scales)."""
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2
    M, K = x.shape
    nc, ns, ne = bs_split_size(fmt, M, K)
    codes = torch.empty(nc, dtype=torch.uint8, device=x.device)
    scales = torch.empty(ns, dtype=torch.uint8, device=x.device)
    x_exp = torch.empty(ne // 4, dtype=torch.int32, device=x.device)
    _check(lib().qgemm_bs_split_x(_fmt(fmt), _ptr(x), M, K, _ptr(codes), _ptr(scales),
                                  _ptr(x_exp), _stream(stream)), "qgemm_bs_split_x")
    return codes, scales, x_exp


def bs_workspace_size(fmt: int, N: int, K: int, M: int) -> int:
    n = _SZ()
    _check(lib().qgemm_bs_workspace_size(fmt, N, K, M, ctypes.byref(n)), "qgemm_bs_workspace_size")
    return n.value


def bs_run(x: torch.Tensor, pw: PackedWeight, y: torch.Tensor | None = None, y_dtype=torch.float32,
           workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """qgemm_bs_run: the block-scaled path (MXFP4, NVFP4 or FP8 weights): x bf16 [M, K] -> y [M, N]."""
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2
    M, K = x.shape
    assert K == pw.K
    if y is None:
        y = torch.empty((M, pw.N), dtype=y_dtype, device=x.device)
    ydt = Y_BF16 if y.dtype == torch.bfloat16 else Y_F32
    if workspace is None:
        nbytes = bs_workspace_size(pw.fmt, pw.N, K, M)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    _check(lib().qgemm_bs_run(pw.fmt, _ptr(x), M, K, _ptr(pw.codes), _ptr(pw.scales),
                              _ptr(pw.tensor_scale), pw.N, _ptr(y), ydt, _ptr(workspace),
                              workspace.numel(), _stream(stream)), "qgemm_bs_run")
    return y


def bs_ffn_workspace_size(fmt, N: int, K: int, M: int) -> int:
    n = _SZ()
    _check(lib().qgemm_bs_ffn_workspace_size(_fmt(fmt), N, K, M, ctypes.byref(n)),
           "qgemm_bs_ffn_workspace_size")
    return n.value


def bs_ffn_gate_up(x: torch.Tensor, wg: PackedWeight, wu: PackedWeight, h: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """qgemm_bs_ffn_gate_up: h = bf16(SiLU(x Wg^T) * (x Wu^T)) on the block-scaled path."""
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous()
    M, K = x.shape
    assert wg.fmt == wu.fmt and wg.N == wu.N and wg.K == wu.K == K
    if h is None:
        h = torch.empty((M, wg.N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(max(bs_ffn_workspace_size(wg.fmt, wg.N, K, M), 16),
                                dtype=torch.uint8, device=x.device)
    _check(lib().qgemm_bs_ffn_gate_up(wg.fmt, _ptr(x), M, K, _ptr(wg.codes), _ptr(wg.scales),
                                      _ptr(wg.tensor_scale), _ptr(wu.codes), _ptr(wu.scales),
                                      _ptr(wu.tensor_scale), wg.N, _ptr(h), _ptr(workspace),
                                      workspace.numel(), _stream(stream)), "qgemm_bs_ffn_gate_up")
    return h


def ffn_gate_up(x: torch.Tensor, wg: PackedWeight, wu: PackedWeight, h: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """qgemm_ffn_gate_up: h = bf16(SiLU(x Wg^T) * (x Wu^T)), x bf16 [M, K] -> h bf16 [M, N]."""
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous()
    M, K = x.shape
    assert wg.fmt == wu.fmt and wg.N == wu.N and wg.K == wu.K == K
    if h is None:
        h = torch.empty((M, wg.N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        nbytes = ffn_workspace_size(wg.fmt, wg.N, K, M)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    _check(lib().qgemm_ffn_gate_up(wg.fmt, _ptr(x), M, K, _ptr(wg.codes), _ptr(wg.scales),
                                   _ptr(wg.tensor_scale), _ptr(wu.codes), _ptr(wu.scales),
                                   _ptr(wu.tensor_scale), wg.N, _ptr(h), _ptr(workspace),
                                   workspace.numel(), _stream(stream)), "qgemm_ffn_gate_up")
    return h


# ---- routed mixture-of-experts --------------------------------------------------------

def moe_workspace_size(fmt, N: int, K: int, M: int, max_rows: int) -> int:
    b = _SZ()
    _check(lib().qgemm_moe_workspace_size(_fmt(fmt), N, K, M, max_rows, ctypes.byref(b)),
           "qgemm_moe_workspace_size")
    return b.value


class ExpertTable:
    """Device pointer tables of a list of packed experts (one PackedWeight each, same format
    and shape): codes, scales (absent for FP8) and tensor scales (NVFP4, FP8)."""

    def __init__(self, experts):
        assert experts and all(e.fmt == experts[0].fmt and e.N == experts[0].N and
                               e.K == experts[0].K for e in experts)
        self.fmt, self.N, self.K, self.E = experts[0].fmt, experts[0].N, experts[0].K, len(experts)
        dev = experts[0].codes.device

        def table(ts):
            return torch.tensor([t.data_ptr() for t in ts], dtype=torch.int64, device=dev)
        self.codes = table([e.codes for e in experts])
        self.scales = table([e.scales for e in experts]) if experts[0].scales.numel() else None
        self.ts = (table([e.tensor_scale for e in experts])
                   if experts[0].tensor_scale is not None else None)
        self.experts = experts  # keeps the buffers alive


def _moe_common(x, offsets, tab):
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2
    assert offsets.is_cuda and offsets.dtype == torch.int32 and offsets.numel() == tab.E + 1
    assert x.shape[1] == tab.K


def moe_run(x: torch.Tensor, offsets: torch.Tensor, tab: ExpertTable, max_rows: int,
            y: torch.Tensor | None = None, y_dtype=torch.float32, workspace=None, stream=None):
    """qgemm_moe_run: rows of x grouped by expert (int32 offsets[E+1] on the device)."""
    _moe_common(x, offsets, tab)
    M, K = x.shape
    if y is None:
        y = torch.empty((M, tab.N), dtype=y_dtype, device=x.device)
    ydt = Y_BF16 if y.dtype == torch.bfloat16 else Y_F32
    if workspace is None:
        nbytes = moe_workspace_size(tab.fmt, tab.N, K, M, max_rows)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    _check(lib().qgemm_moe_run(tab.fmt, _ptr(x), M, K, tab.E, _ptr(offsets), max_rows,
                               _ptr(tab.codes), _ptr(tab.scales), _ptr(tab.ts), tab.N, _ptr(y), ydt,
                               _ptr(workspace), workspace.numel(), _stream(stream)), "qgemm_moe_run")
    return y


def moe_gate_up(x: torch.Tensor, offsets: torch.Tensor, gate: ExpertTable, up: ExpertTable,
                max_rows: int, h: torch.Tensor | None = None, workspace=None, stream=None):
    """qgemm_moe_gate_up: h = bf16(SiLU(x Wg_e^T) * (x Wu_e^T)) per routed row."""
    _moe_common(x, offsets, gate)
    assert gate.fmt == up.fmt and gate.N == up.N and gate.K == up.K and gate.E == up.E
    M, K = x.shape
    if h is None:
        h = torch.empty((M, gate.N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        nbytes = moe_workspace_size(gate.fmt, gate.N, K, M, max_rows)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    _check(lib().qgemm_moe_gate_up(gate.fmt, _ptr(x), M, K, gate.E, _ptr(offsets), max_rows,
                                   _ptr(gate.codes), _ptr(gate.scales), _ptr(gate.ts),
                                   _ptr(up.codes), _ptr(up.scales), _ptr(up.ts), gate.N, _ptr(h),
                                   _ptr(workspace), workspace.numel(), _stream(stream)),
           "qgemm_moe_gate_up")
    return h
