"""GPU parity of qgemm_pack / qgemm_run against the CPU oracle, through the C ABI.

Bars: packing is byte-exact; GEMM results are within 1e-3 normalised error
(max |y - y_ref| / (||x_b|| ||w_n||)); one-hot inputs reproduce dequantised columns exactly
(after the operand rounding of Q8_0); rows are bit-identical across widths 1..256 (the
hipfire PR's chunked-vs-unchunked boundary matrix, generalised)."""
import numpy as np
import pytest
import torch

import oracle
from block_quantized_weight_qgemm_b200 import inputs
from block_quantized_weight_qgemm_b200 import qgemm

from gpu_helpers import TOL, Case, gpu_run, norm_err, round_bf16, round_f16, tile_packed, x_bits

pytestmark = pytest.mark.gpu

FMTS = ["q8_0", "nvfp4", "mxfp4", "fp8"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_quantized_weight_qgemm_b200 import build
    build.build()
    qgemm.lib()
    qgemm.device_status(reset=True)
    yield
    assert qgemm.device_status(reset=True) == qgemm.OK


def _specials(N, K, seed):
    W = inputs.weights(N, K, seed=seed).numpy().copy()
    W[0, :64] = 0.0
    W[1, 32:64] *= 1e-5
    W[2, :16] = np.float32(0.015)
    W[3, 64:96] *= 40.0
    W[N - 1, K - 32:] = -W[N - 1, K - 32:]
    return W


# --------------------------------------------------------------------------------------
# qgemm_pack
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", [(300, 512), (512, 1024), (129, 2048)])
def test_pack_byte_exact(fmt, N, K):
    W = _specials(N, K, 40 + N)
    codes_rm, scales_rm, ts = oracle.pack(fmt, W)
    codes, scales = tile_packed(fmt, codes_rm, scales_rm, N, K)
    pw = qgemm.pack(fmt, torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    gc, gs = pw.codes.cpu().numpy(), pw.scales.cpu().numpy()
    mism = np.argwhere(gc != codes)
    assert mism.size == 0, "codes differ at %s: gpu %s oracle %s" % (
        mism[:5].tolist(), gc[tuple(mism[0])], codes[tuple(mism[0])])
    mism = np.argwhere(gs != scales)
    assert mism.size == 0, "scales differ at %s" % mism[:5].tolist()
    if fmt in ("nvfp4", "fp8"):
        assert pw.tensor_scale.item() == ts


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", [(300, 512), (129, 1056)])
def test_repack_rowmajor_matches_layout(fmt, N, K):
    if fmt != "nvfp4" and K % 32:
        pytest.skip("K must be a multiple of 32")
    W = _specials(N, K, 60 + N)
    codes_rm, scales_rm, ts = oracle.pack(fmt, W)
    ct, st = tile_packed(fmt, codes_rm, scales_rm, N, K)
    pw = qgemm.repack_rowmajor(fmt, torch.from_numpy(codes_rm).cuda(),
                               torch.from_numpy(scales_rm).cuda(), N, K)
    torch.cuda.synchronize()
    assert np.array_equal(pw.codes.cpu().numpy(), ct)
    assert np.array_equal(pw.scales.cpu().numpy(), st)


# --------------------------------------------------------------------------------------
# qgemm_run parity
# --------------------------------------------------------------------------------------
@pytest.fixture(scope="module")
def small_cases():
    # 300 rows = 2 full 128-row tiles + a ragged tail; K = 1024 spans several weight stages
    return {f: Case(f, 300, 1024, seed=7) for f in FMTS}


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("B", [1, 5, 16, 17, 64, 65, 130, 256, 257, 300, 520])
def test_run_parity_small(small_cases, fmt, B):
    case = small_cases[fmt]
    x = inputs.activations(B, case.K, seed=8)
    xb = x_bits(x)
    y_ref = oracle.gemm(xb, case.Wd)
    y = gpu_run(case, x)
    err = norm_err(y, y_ref, xb, case.Wd)
    assert err <= TOL, "normalised error %.3e" % err
    yb = gpu_run(case, x, torch.bfloat16)
    errb = norm_err(yb, y_ref, xb, case.Wd)
    assert errb <= TOL, "bf16 output: normalised error %.3e" % errb
    # bf16 output is the fp32 result rounded once
    assert np.array_equal(yb, round_bf16(y))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("B", [8, 300])  # f16 operand path and bf16 operand path
def test_run_one_hot_exact(small_cases, fmt, B):
    case = small_cases[fmt]
    K = case.K
    cols = [(37 * i + 5) % K for i in range(B)]
    cols[:4] = [0, 1, K - 1, K - 2]
    x = inputs.one_hot(B, K, cols)
    y = gpu_run(case, x)
    expect = case.Wd[:, cols].T.copy()
    if fmt == "q8_0":
        # the weight operand holds q*d rounded once to the 16-bit operand type
        expect = round_f16(expect) if B <= 256 else round_bf16(expect)
    else:
        expect = expect.astype(np.float32).astype(np.float64)  # only the fp32 tensor-scale rounding
    bad = np.argwhere(y != expect)
    assert bad.size == 0, "first mismatches (b, n): %s gpu %r expect %r" % (
        bad[:4].tolist(), y[tuple(bad[0])], expect[tuple(bad[0])])


@pytest.mark.parametrize("fmt", FMTS)
def test_run_row_sums(small_cases, fmt):
    case = small_cases[fmt]
    x = torch.ones(3, case.K, dtype=torch.bfloat16)
    y = gpu_run(case, x)
    y_ref = oracle.gemm(x_bits(x), case.Wd)
    assert norm_err(y, y_ref, x_bits(x), case.Wd) <= TOL


def test_run_special_rows():
    # zero rows, a row with one huge element, a tiny row: power-of-two x rescaling keeps them exact
    case = Case("nvfp4", 256, 512, seed=9)
    x = inputs.activations(6, 512, seed=10)
    x[0] = 0
    x[1, 7] = 3.0e38
    x[2] *= 1e-30
    x[3, :] = 60000.0
    x[4, ::2] = -1e-35
    xb = x_bits(x)
    y_ref = oracle.gemm(xb, case.Wd)
    y = gpu_run(case, x)
    for b in range(6):
        if b == 1:
            continue  # 3e38 * w overflows fp32 in any accumulation order
        err = norm_err(y[b:b + 1], y_ref[b:b + 1], xb[b:b + 1], case.Wd)
        assert err <= TOL, (b, err)
    assert np.all(y[0] == 0.0)


@pytest.mark.parametrize("fmt", FMTS)
def test_run_extreme_rows_f16_path(small_cases, fmt):
    # rows at the ends of the bf16 range (widths <= 256 convert x to f16 after a per-row power
    # of two): a maximum of 1e-36 (the row's scale 2^-e exceeds 2^127), bf16 subnormals only,
    # the largest finite magnitude beside values near the smallest normal, and a zero row
    case = small_cases[fmt]
    K = case.K
    x = inputs.activations(7, K, seed=15).float()
    x[0] *= 1e-36 / x[0].abs().max()
    sub = np.array([0x0001, 0x0003, 0x007F, 0x8005, 0x0040, 0x8001], dtype=np.uint16)
    x[1] = inputs.bits_to_bf16(np.resize(sub, K)).float()
    x[2, ::3] = 1e-38
    x[2, 1::3] = -2e-38
    x[2, 5] = 3.0e38
    x[3] = 0.0
    x[4, ::2] *= 2.0 ** -100
    x[5, 17] = -3.0e38
    x[5, 18] = 2.5e38
    x = x.to(torch.bfloat16)
    xb = x_bits(x)
    y_ref = oracle.gemm(xb, case.Wd)
    y = gpu_run(case, x)
    assert np.isfinite(y).all()
    for b in range(7):
        err = norm_err(y[b:b + 1], y_ref[b:b + 1], xb[b:b + 1], case.Wd)
        assert err <= TOL, (b, err)
    assert np.all(y[3] == 0.0)
    # bf16 output is still the fp32 result rounded once
    assert np.array_equal(gpu_run(case, x, torch.bfloat16), round_bf16(y))


# --------------------------------------------------------------------------------------
# batch invariance (bit-exact), the boundary matrix of the hipfire PR generalised
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("fmt", FMTS)
def test_batch_invariance_small(small_cases, fmt, golden):
    case = small_cases[fmt]
    x = inputs.activations(256 + 40, case.K, seed=11)
    full = gpu_run(case, x[:256])
    widths = sorted(set([1, 2, 4, 5, 8, 9, 15, 16, 17, 31, 32, 33, 48, 63, 64, 65, 70, 76, 96,
                         127, 128, 129, 192, 200, 255, 256] + golden("q8_boundary_matrix.json")["widths"]))
    for B in widths:
        y = gpu_run(case, x[:B])
        assert np.array_equal(y, full[:B]), "width %d differs from width 256" % B
    # shifted windows: row r computed at other positions of the batch tile
    for s0, B in [(1, 64), (7, 70), (40, 256), (63, 1), (100, 65)]:
        y = gpu_run(case, x[s0:s0 + B])
        ref = gpu_run(case, x[s0:s0 + 256])[:B] if s0 + 256 <= x.shape[0] else None
        if s0 + B <= 256:
            assert np.array_equal(y, full[s0:s0 + B]), (s0, B)
        if ref is not None:
            assert np.array_equal(y, ref), (s0, B)
    # the chunked decompositions of the PR: 70 = 64 + 6 and 256 = 4 x 64
    parts = np.concatenate([gpu_run(case, x[o:o + p]) for o, p in [(0, 64), (64, 6)]])
    assert np.array_equal(parts, full[:70])
    parts = np.concatenate([gpu_run(case, x[o:o + 64]) for o in range(0, 256, 64)])
    assert np.array_equal(parts, full)


def test_tiny_q8_config(golden):
    """Q8_0 W[512, 1024] ~ N(0, 0.02), x bf16 [B, 1024] ~ N(0, 1), seed 0; B in {1,63,64,65,70,76}."""
    case = Case("q8_0", 512, 1024, seed=inputs.W_SEED)
    x = inputs.activations(76, 1024, seed=inputs.X_SEED)
    xb = x_bits(x)
    y_ref = oracle.gemm(xb, case.Wd)
    full = gpu_run(case, x)
    assert norm_err(full, y_ref, xb, case.Wd) <= TOL
    for B in (1, 63, 64, 65, 70):
        y = gpu_run(case, x[:B])
        assert np.array_equal(y, full[:B]), B
        assert norm_err(y, y_ref[:B], xb[:B], case.Wd) <= TOL


# --------------------------------------------------------------------------------------
# host-side errors on a real device
# --------------------------------------------------------------------------------------
def test_errors_on_device(small_cases):
    import ctypes
    case = small_cases["q8_0"]
    x = inputs.activations(64, case.K, seed=12).cuda()
    y = torch.empty(64, case.N, device="cuda")
    need = qgemm.workspace_size("q8_0", case.N, case.K, 64)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    lib = qgemm.lib()
    st = lib.qgemm_run(0, x.data_ptr(), 64, case.K, case.pw.codes.data_ptr(),
                       case.pw.scales.data_ptr(), None, case.N, y.data_ptr(), 0,
                       ws.data_ptr(), need - 1 if need > 0 else 0, None)
    assert st == (6 if need > 0 else 0)
    st = lib.qgemm_run(0, x.data_ptr() + 2, 64, case.K, case.pw.codes.data_ptr(),
                       case.pw.scales.data_ptr(), None, case.N, y.data_ptr(), 0,
                       ws.data_ptr(), need, None)
    assert st == 5
    torch.cuda.synchronize()


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("B", [3, 300])
def test_run_ragged_k(fmt, B):
    # K = 1056: the last weight chunk is partial (8.25 Q8_0 chunks, 4.125 FP4 chunks); N = 200
    case = Case(fmt, 200, 1056, seed=13)
    x = inputs.activations(B, 1056, seed=14)
    xb = x_bits(x)
    y_ref = oracle.gemm(xb, case.Wd)
    err = norm_err(gpu_run(case, x), y_ref, xb, case.Wd)
    assert err <= TOL, err
