"""GPU parity of the block-scaled path for MXFP4, NVFP4 and FP8 weights (qgemm_bs_split_x /
qgemm_bs_run) against the CPU oracle, through the C ABI.

Bars:
  * the split of x is exact: the sum of the terms the GPU writes (three E2M1 terms for FP4
    weights, two E4M3 terms for FP8; decoded on the host from the layout of include/qgemm.h)
    equals oracle.split_x_bs bit for bit;
  * the GEMM is the product of that split with the dequantised weights up to fp32
    accumulation (normalised error 2e-5), and within the method's 1e-3 of the exact product
    at K >= 1024 (the split's own residual is measured in the oracle pins);
  * one-hot rows of x reproduce the dequantised weight columns exactly.
Shapes span several tiles with ragged M, N and K tails, both tilings (up to 128 rows the
weights are the MMA M operand and K is split over the SMs; above, x is), and the 27B shapes at
prefill and decode widths on sampled rows."""
import numpy as np
import pytest
import torch

import oracle
from block_quantized_weight_qgemm_b200 import inputs
from block_quantized_weight_qgemm_b200 import qgemm
from gpu_helpers import TOL, Case, norm_err, x_bits

pytestmark = pytest.mark.gpu

SPLIT_TOL = 2e-5  # fp32 accumulation of exact E2M1 x E2M1 products (K u bounds it by 1.2e-4)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_quantized_weight_qgemm_b200 import build
    build.build()
    qgemm.lib()
    qgemm.device_status(reset=True)
    yield
    assert qgemm.device_status(reset=True) == qgemm.OK


# per weight format: terms, K per chunk, block, scale bytes per row and chunk
SPLIT_GEOM = {"mxfp4": (3, 256, 32, 8), "nvfp4": (3, 256, 16, 16), "fp8": (2, 128, 32, 4)}


def _decode_split(fmt, codes, scales, x_exp, M, K):
    """Sum of the terms per element, from the documented layout (numpy only)."""
    terms, ck, blk, sbr = SPLIT_GEOM[fmt]
    C, Mt = -(-K // ck), -(-M // 128)
    svals = (np.array([oracle.e4m3(b) if b < 0x7F else 0.0 for b in range(256)]) if fmt == "nvfp4"
             else np.exp2(np.arange(256, dtype=np.float64) - 127.0))
    cb = codes.reshape(Mt, C, terms, 128, 8, 16)
    un = np.empty_like(cb)
    for r in range(128):
        for g in range(8):
            un[:, :, :, r, g, :] = cb[:, :, :, r, g ^ (r & 7), :]
    un = un.reshape(Mt, C, terms, 128, 128)
    if fmt == "fp8":  # one E4M3 code per byte
        vals = np.array([oracle.e4m3(b) for b in range(256)])
        el = un
    else:             # two E2M1 codes per byte, the even element in the low nibble
        vals = np.array([oracle.e2m1(c) for c in range(16)])
        el = np.stack([un & 15, un >> 4], axis=-1).reshape(Mt, C, terms, 128, 256)
    sc = scales.reshape(Mt, C, terms, 128, sbr)
    val = vals[el] * np.repeat(svals[sc], blk, axis=-1)
    tot = val.sum(axis=2).transpose(0, 2, 1, 3).reshape(Mt * 128, C * ck)
    return tot, tot[:M, :K] * np.exp2(x_exp[:M].astype(np.float64))[:, None]


def _special_rows(x: torch.Tensor) -> torch.Tensor:
    """Rows 0..5 (as far as x has them) replaced by edge cases; a one-row x keeps its row."""
    x = x.clone()
    M, K = x.shape
    if M < 6:
        return x
    x[0] = 0.0                                        # all-zero row
    x[1] = x[1] * 1e-30                                # tiny row (x_exp near -100)
    x[2, : K // 2] = x[2, : K // 2] * 1e20             # blocks 2^66 apart in one row
    x[3, 32:64] = 0.0                                  # a zero block
    x[4, ::7] = -x[4, ::7] * 3.0e4                     # mixed signs and magnitudes
    x[5, :] = 6.0                                      # exactly representable in one term
    return x


FMTS = ["mxfp4", "nvfp4", "fp8"]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,K", [(1, 32), (130, 288), (257, 1024), (200, 5120)])
def test_split_bit_exact(fmt, M, K):
    x = _special_rows(inputs.activations(M, K, seed=20 + M))
    if M >= 7:
        x[6] = x[6] * 2.0 ** -128  # bf16 subnormals: 2^-x_exp is past the normal range
    codes, scales, x_exp = qgemm.bs_split_x(x.cuda(), fmt)
    torch.cuda.synchronize()
    codes, scales, x_exp = codes.cpu().numpy(), scales.cpu().numpy(), x_exp.cpu().numpy()
    full, xs_gpu = _decode_split(fmt, codes, scales, x_exp, M, K)
    xs = oracle.split_x_bs(x_bits(x), fmt)
    bad = np.argwhere(xs_gpu != xs)
    assert bad.size == 0, "split differs at %s: gpu %r oracle %r" % (
        bad[:4].tolist(), xs_gpu[tuple(bad[0])], xs[tuple(bad[0])])
    # padding rows and columns hold zeros
    assert not full[M:].any() and not full[:, K:].any()
    assert (x_exp[M:] == 0).all()


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K", [(1, 300, 512), (16, 256, 256), (33, 1000, 1056),
                                   (128, 640, 4096), (128, 256, 256), (300, 400, 320),
                                   (129, 1000, 1056), (517, 300, 2048)])
def test_gemm_is_the_split_product(fmt, M, N, K):
    case = Case(fmt, N, K, seed=30 + N)
    x = _special_rows(inputs.activations(M, K, seed=31 + M))
    y = qgemm.bs_run(x.cuda(), case.pw)
    torch.cuda.synchronize()
    y = y.cpu().numpy().astype(np.float64)
    xb = x_bits(x)
    ys = oracle.gemm_f64(oracle.split_x_bs(xb, fmt), case.Wd)
    assert norm_err(y, ys, xb, case.Wd) <= SPLIT_TOL
    if K >= 1024:
        assert norm_err(y, oracle.gemm(xb, case.Wd), xb, case.Wd) <= TOL


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [256, 64])
def test_one_hot_rows_give_weight_columns(fmt, M):
    N, K = 512, 768
    case = Case(fmt, N, K, seed=41)
    ks = (np.arange(M) * 37 + 3) % K
    x = torch.zeros(M, K, dtype=torch.bfloat16)
    x[np.arange(M), ks] = 1.0
    x[7, ks[7]] = -0.375  # exactly one term: -1.5 * 2^-2
    y = qgemm.bs_run(x.cuda(), case.pw).cpu().numpy()
    exp = case.Wd[:, ks].T.copy()
    exp[7] *= -0.375
    # one exact product per output (times the NVFP4 / FP8 tensor scale, rounded once to fp32)
    assert np.array_equal(y, exp.astype(np.float32))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [300, 40])
def test_bf16_output_and_workspace_reuse(fmt, M):
    N, K = 640, 1024
    case = Case(fmt, N, K, seed=43)
    x = inputs.activations(M, K, seed=44).cuda()
    ws = torch.empty(qgemm.bs_workspace_size(qgemm._fmt(fmt), N, K, M), dtype=torch.uint8,
                     device="cuda")
    y32 = qgemm.bs_run(x, case.pw, workspace=ws)
    y16 = qgemm.bs_run(x, case.pw, y_dtype=torch.bfloat16, workspace=ws)
    y32b = qgemm.bs_run(x, case.pw, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y32, y32b)  # deterministic
    assert torch.equal(y16, y32.to(torch.bfloat16))


@pytest.mark.parametrize("fmt,N,K,M", [("mxfp4", 17408, 5120, 2048), ("mxfp4", 5120, 17408, 2048),
                                       ("mxfp4", 17408, 5120, 32), ("mxfp4", 5120, 17408, 32),
                                       ("nvfp4", 17408, 5120, 2048), ("nvfp4", 17408, 5120, 16),
                                       ("nvfp4", 5120, 17408, 16), ("fp8", 17408, 5120, 2048),
                                       ("fp8", 5120, 17408, 2048), ("fp8", 17408, 5120, 32)])
def test_27b_prefill_sampled_rows(fmt, N, K, M):
    case = Case(fmt, N, K, seed=inputs.W_SEED if N == 17408 else inputs.W3_SEED)
    x = inputs.activations(M, K, seed=50)
    y = qgemm.bs_run(x.cuda(), case.pw)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 127, 128, 1000, M - 1]) if M > 1000 else np.array([0, 1, M // 2, M - 1])
    y = y.cpu().numpy()[rows].astype(np.float64)  # rows picked on the host
    xb = x_bits(x)[rows]
    ys = oracle.gemm_f64(oracle.split_x_bs(xb, fmt), case.Wd)
    assert norm_err(y, ys, xb, case.Wd) <= SPLIT_TOL
    assert norm_err(y, oracle.gemm(xb, case.Wd), xb, case.Wd) <= TOL


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [40, 300, 2100])
def test_fused_gate_up(fmt, M):
    # h = bf16(SiLU(g) * u) with g, u the split's products: one bf16 ulp plus the split bar
    # propagated to first order (the chunk of 2048 rows is crossed at M = 2100)
    from gpu_helpers import bf16_bits_of, h_bound_violations
    N, K = 640, 1024
    cg, cu = Case(fmt, N, K, seed=71), Case(fmt, N, K, seed=72)
    x = inputs.activations(M, K, seed=73)
    x[0] = 0.0          # an all-zero row
    x[1] = x[1] * 1e-4  # a small row (h in the linear part of SiLU)
    h = qgemm.bs_ffn_gate_up(x.cuda(), cg.pw, cu.pw)
    torch.cuda.synchronize()
    xb = x_bits(x)
    rows = np.arange(M) if M <= 300 else np.array([0, 1, 5, 1000, 2047, 2048, M - 1])
    xs = oracle.split_x_bs(xb[rows], fmt)
    g = oracle.gemm_f64(xs, cg.Wd)
    u = oracle.gemm_f64(xs, cu.Wd)
    bad, worst = h_bound_violations(bf16_bits_of(h)[rows], g, u, xb[rows], cg.Wd, cu.Wd, tol=SPLIT_TOL)
    assert bad == 0, "%d outputs outside the bound (worst ratio %.2f)" % (bad, worst)
