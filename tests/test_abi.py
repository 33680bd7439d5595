"""C-ABI checks that need no GPU: the library loads, exports every entry point the header
declares, and its host-side logic (validation, sizes, the K-split rule) behaves as documented.
No compute is launched."""
import ctypes
import os
import re

import pytest

import oracle
from block_quantized_weight_qgemm_b200 import build as qbuild
from block_quantized_weight_qgemm_b200 import qgemm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qgemm.h")


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return qgemm.lib()


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qgemm_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    # and the binding covers exactly the header's entry points
    assert sorted(n for n, _, _ in qgemm.SIGNATURES) == names


def test_status_strings(lib):
    for code in range(11):
        s = lib.qgemm_status_str(code).decode()
        assert s and s != "unknown status"
    assert lib.qgemm_status_str(99).decode() == "unknown status"
    assert lib.qgemm_last_cuda_error().decode() == ""


@pytest.mark.parametrize("fmt", ["q8_0", "nvfp4", "mxfp4", "fp8"])
@pytest.mark.parametrize("K", [32, 64, 96, 1024, 5120, 17408])
def test_pitches_match_layout_spec(lib, fmt, K):
    if fmt in ("q8_0", "mxfp4") and K % 32:
        pytest.skip("K must be a multiple of 32")
    cp, sp = qgemm.row_pitches(fmt, K)
    assert (cp, sp) == (oracle.code_pitch(fmt, K), oracle.scale_pitch(fmt, K))
    T, C, CK, SB = qgemm.packed_geometry(fmt, 300, K)
    byte_codes = fmt in ("q8_0", "fp8")
    assert T == 3 and CK == (128 if byte_codes else 256) and C == -(-K // CK)
    assert SB == {"q8_0": 8, "nvfp4": 16, "mxfp4": 8, "fp8": 0}[fmt]
    cb, sb = qgemm.packed_size(fmt, 300, K)
    assert (cb, sb) == (T * C * 128 * 128, T * C * 128 * SB)
    # the tiled layout holds every byte of the row-major packing (plus zero padding)
    assert cb >= 300 * (K if byte_codes else K // 2)


def test_argument_errors(lib):
    sz = ctypes.c_size_t()
    i64 = ctypes.c_int64()
    assert lib.qgemm_packed_size(5, 4, 32, ctypes.byref(sz), ctypes.byref(sz)) == 1   # format
    assert lib.qgemm_packed_size(0, 0, 32, ctypes.byref(sz), ctypes.byref(sz)) == 2   # N < 1
    assert lib.qgemm_packed_size(0, 4, 0, ctypes.byref(sz), ctypes.byref(sz)) == 2    # K < 1
    assert lib.qgemm_packed_size(0, 4, 48, ctypes.byref(sz), ctypes.byref(sz)) == 3   # K % 32
    assert lib.qgemm_packed_size(1, 4, 40, ctypes.byref(sz), ctypes.byref(sz)) == 3   # K % 16
    assert lib.qgemm_packed_size(1, 4, 48, ctypes.byref(sz), ctypes.byref(sz)) == 0
    assert lib.qgemm_packed_size(0, 4, 32, None, None) == 4                           # NULL
    assert lib.qgemm_row_pitches(2, 48, ctypes.byref(i64), ctypes.byref(i64)) == 3
    assert lib.qgemm_workspace_size(0, 4, 32, 0, ctypes.byref(sz)) == 2               # B < 1
    # qgemm_run: validation happens before any device work
    assert lib.qgemm_run(0, None, 4, 64, None, None, None, 8, None, 0, None, 0, None) == 4
    assert lib.qgemm_run(0, 16, 4, 64, 16, 16, None, 8, 16, 7, None, 0, None) == 1   # y dtype
    assert lib.qgemm_run(1, 16, 4, 64, 16, 16, None, 8, 16, 0, None, 0, None) == 4   # NVFP4 ts
    assert lib.qgemm_run(0, 8, 4, 64, 16, 16, None, 8, 16, 0, None, 0, None) == 5    # misaligned
    assert lib.qgemm_run(0, 16, 0, 64, 16, 16, None, 8, 16, 0, None, 0, None) == 2   # B = 0
    assert lib.qgemm_pack(0, None, 4, 64, None, None, None, None) == 4
    # FP8: no block scales (NULL accepted) but the tensor scale is required
    assert lib.qgemm_run(3, 16, 4, 64, 16, None, None, 8, 16, 0, None, 0, None) == 4
    assert lib.qgemm_packed_size(3, 4, 40, ctypes.byref(sz), ctypes.byref(sz)) == 3   # K % 16
    assert lib.qgemm_packed_size(3, 4, 48, ctypes.byref(sz), ctypes.byref(sz)) == 0
    assert sz.value == 0                                                              # no scales
    assert lib.qgemm_packed_size(4, 4, 48, ctypes.byref(sz), ctypes.byref(sz)) == 1   # format
    assert lib.qgemm_ffn_gate_up(0, 16, 4, 64, 16, 16, None, None, 16, None, 8, 16, None, 0,
                                 None) == 4
    # routed experts: argument checks before any device work
    assert lib.qgemm_moe_run(0, 16, 4, 64, 2, None, 4, 16, 16, None, 8, 16, 0, None, 0,
                             None) == 4                                             # offsets
    assert lib.qgemm_moe_run(0, 16, 4, 64, 0, 16, 4, 16, 16, None, 8, 16, 0, None, 0,
                             None) == 2                                             # E = 0
    assert lib.qgemm_moe_run(1, 16, 4, 64, 2, 16, 4, 16, 16, None, 8, 16, 0, None, 0,
                             None) == 4                                             # NVFP4 ts table
    assert lib.qgemm_moe_run(0, 16, 4, 64, 2, 16, 4, 20, 16, None, 8, 16, 0, None, 0,
                             None) == 5                                             # table alignment
    assert lib.qgemm_moe_gate_up(3, 16, 4, 64, 2, 16, 4, 16, None, 16, 16, None, None, 8, 16,
                                 None, 0, None) == 4                                # up ts table


def test_block_scaled_argument_errors(lib):
    sz = ctypes.c_size_t()
    # the block-scaled path takes MXFP4, NVFP4 and FP8 weights, and checks before any device work
    for fmt in (0, 7):
        assert lib.qgemm_bs_workspace_size(fmt, 256, 256, 128, ctypes.byref(sz)) == 1
        assert lib.qgemm_bs_run(fmt, 16, 4, 64, 16, 16, 16, 8, 16, 0, 16, 1 << 20, None) == 1
    assert lib.qgemm_bs_workspace_size(2, 256, 48, 128, ctypes.byref(sz)) == 3      # K % 32
    assert lib.qgemm_bs_workspace_size(2, 256, 256, 0, ctypes.byref(sz)) == 2       # M < 1
    assert lib.qgemm_bs_run(2, None, 4, 64, 16, 16, None, 8, 16, 0, 16, 1 << 20, None) == 4
    assert lib.qgemm_bs_run(2, 8, 4, 64, 16, 16, None, 8, 16, 0, 16, 1 << 20, None) == 5
    assert lib.qgemm_bs_run(2, 16, 4, 64, 16, 16, None, 8, 16, 0, 16, 16, None) == 6  # workspace
    assert lib.qgemm_bs_run(1, 16, 4, 64, 16, 16, None, 8, 16, 0, 16, 1 << 20, None) == 4  # NVFP4 ts
    assert lib.qgemm_bs_run(3, 16, 4, 64, 16, None, None, 8, 16, 0, 16, 1 << 20, None) == 4  # FP8 ts
    assert lib.qgemm_bs_split_x(2, 16, 4, 48, 16, 16, 16, None) == 3                 # K % 32
    assert lib.qgemm_bs_split_x(2, 16, 4, 64, None, 16, 16, None) == 4
    assert lib.qgemm_bs_split_x(0, 16, 4, 64, 16, 16, 16, None) == 1                 # format
    c, s, e = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    for fmt, chunks, terms, sbr in ((2, 2, 3, 8), (1, 2, 3, 16), (3, 3, 2, 4)):
        assert lib.qgemm_bs_split_size(fmt, 300, 320, ctypes.byref(c), ctypes.byref(s),
                                       ctypes.byref(e)) == 0
        # 3 token tiles x chunks (of 256 K, 128 for FP8) x terms of 128 x 128 code bytes and
        # 128 x sbr scale bytes
        n = 3 * chunks * terms
        assert (c.value, s.value, e.value) == (n * 16384, n * 128 * sbr, 3 * 128 * 4)
        assert lib.qgemm_bs_workspace_size(fmt, 256, 320, 300, ctypes.byref(sz)) == 0
        assert sz.value == c.value + s.value + e.value


def test_no_width_limit_in_sizes(lib):
    # every width has a workspace size; nothing is rejected above 64 (the pages' MAX_BATCH)
    for B in (1, 63, 64, 65, 70, 76, 255, 256, 257, 1000, 8192):
        assert qgemm.workspace_size("q8_0", 17408, 5120, B) >= 0


def test_split_rule_depends_only_on_shape(lib):
    # the K split is a function of (format, N, K): pinned values for the 27B FFN shapes
    got = {(f, N, K): qgemm.split_k(f, N, K) for f in ("q8_0", "nvfp4", "mxfp4")
           for (N, K) in ((17408, 5120), (5120, 17408), (512, 1024))}
    for (f, N, K), s in got.items():
        assert 1 <= s <= 16
    assert got[("q8_0", 17408, 5120)] == 1
    assert got[("nvfp4", 17408, 5120)] == 1
    assert got[("q8_0", 5120, 17408)] == 3
    assert got[("nvfp4", 5120, 17408)] == 3
    # workspace grows with B but the split does not
    w64 = qgemm.workspace_size("q8_0", 5120, 17408, 64)
    w65 = qgemm.workspace_size("q8_0", 5120, 17408, 65)
    assert w65 > w64


def test_prefill_path_needs_no_workspace(lib):
    assert qgemm.workspace_size("nvfp4", 17408, 5120, 2048) == 0


def test_wide_fused_ffn_workspace_holds_g_and_u_of_one_chunk(lib):
    # above 256 rows the fused gate+up runs, per chunk of rows, two plain GEMMs into fp32
    # g and u and one SiLU pass; chunks of 2048 rows, balanced (multiples of 8 rows) only
    # when a full-chunk split would leave a last chunk of 256 rows or fewer
    N = 17408
    assert qgemm.ffn_workspace_size("nvfp4", N, 5120, 2048) == 2 * 2048 * N * 4
    assert qgemm.ffn_workspace_size("nvfp4", N, 5120, 2049) == 2 * 1032 * N * 4
    assert qgemm.ffn_workspace_size("nvfp4", N, 5120, 7235) == 2 * 2048 * N * 4
    assert qgemm.ffn_workspace_size("q8_0", N, 5120, 300) == 2 * 304 * N * 4
    # at or below 256 rows the single fused kernel runs
    assert qgemm.ffn_workspace_size("q8_0", N, 5120, 256) < 256 * N * 4


def test_moe_workspace_holds_f16_rows(lib):
    # routed experts: the f16 copy of all M rows (row pitch K rounded up to 64) and their
    # exponents, 256-byte aligned pieces; none on the wide path
    M, K = 480, 2048
    assert qgemm.moe_workspace_size("nvfp4", 512, K, M, 25) == M * K * 2 + (M * 4 + 255) // 256 * 256
    assert qgemm.moe_workspace_size("nvfp4", 512, K, M, 300) == 0
