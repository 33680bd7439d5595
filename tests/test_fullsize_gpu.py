"""Parity at the 27B-class shapes (hidden 5120, FFN 17408), in the launch configuration the
benchmark times.  The oracle computes sampled output rows one by one (all N columns of each);
batch invariance is checked bit for bit on the full outputs.

Workloads (seeded, synthetic; weights ~N(0, 0.02), activations bf16 ~N(0, 1)):
  Q8_0 gate/up [17408, 5120] and down [5120, 17408], widths 1..256 and 257;
  NVFP4 verify widths B in {1, 4, 5, 8, 9, 16} on [17408, 5120];
  FP8 (E4M3) verify and decode widths, the down shape and an M = 2048 chunk;
  NVFP4 prefill FFN chunk, M in {2048, 7235}: fused gate+up -> h -> down;
  MXFP4 serving mix: B = 32 decode and an M = 8192 prefill chunk on both shapes."""
import numpy as np
import pytest
import torch

import oracle
from block_quantized_weight_qgemm_b200 import inputs
from block_quantized_weight_qgemm_b200 import qgemm
from gpu_helpers import TOL, Case, bf16_bits_of, h_bound_violations, norm_err, tile_packed

pytestmark = pytest.mark.gpu

HIDDEN, INTER = 5120, 17408


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_quantized_weight_qgemm_b200 import build
    build.build()
    qgemm.lib()
    qgemm.device_status(reset=True)
    yield
    assert qgemm.device_status(reset=True) == qgemm.OK


def _run(case, x, ydt=torch.float32):
    y = qgemm.run(x, case.pw, y_dtype=ydt)
    torch.cuda.synchronize()
    return y


def _np(y):
    return y.float().cpu().numpy().astype(np.float64)


def _check_rows(case, y_gpu, x_bits, rows):
    y_ref = oracle.gemm(x_bits[rows], case.Wd)
    err = norm_err(y_gpu[rows], y_ref, x_bits[rows], case.Wd)
    assert err <= TOL, "normalised error %.3e" % err
    return err


@pytest.mark.parametrize("N,K", [(INTER, HIDDEN), (HIDDEN, INTER)])
def test_q8_27b_width_sweep(N, K):
    case = Case("q8_0", N, K, seed=inputs.W_SEED if N == INTER else inputs.W3_SEED)
    # the device packer gives the oracle's bytes at full size too
    pw = qgemm.pack("q8_0", torch.from_numpy(case.W).cuda())
    torch.cuda.synchronize()
    ct, st = tile_packed("q8_0", case.codes, case.scales, N, K)
    assert np.array_equal(pw.codes.cpu().numpy(), ct)
    assert np.array_equal(pw.scales.cpu().numpy(), st)
    del pw

    x = inputs.activations(257, K, seed=inputs.X_SEED).cuda()
    xb = inputs.bf16_bits(x.cpu())
    full = _np(_run(case, x[:256]))
    _check_rows(case, full, xb, [0, 1, 63, 64, 65, 69, 75, 128, 255])
    for B in (1, 2, 8, 16, 63, 64, 65, 70, 76, 128, 200):
        assert np.array_equal(_np(_run(case, x[:B])), full[:B]), "width %d differs from 256" % B
    # bf16 output: the fp32 result rounded once, and batch invariant as well
    fb = _run(case, x[:256], torch.bfloat16)
    assert np.array_equal(_np(fb), _np(torch.from_numpy(full).to(torch.bfloat16)))
    assert np.array_equal(_np(_run(case, x[:65], torch.bfloat16)), _np(fb)[:65])
    # above 256 the bf16-operand path: parity only
    y257 = _np(_run(case, x))
    _check_rows(case, y257, xb, [0, 100, 255, 256])


def test_nvfp4_verify_widths():
    case = Case("nvfp4", INTER, HIDDEN)
    x = inputs.activations(16, HIDDEN, seed=inputs.X_SEED).cuda()
    xb = inputs.bf16_bits(x.cpu())
    full = _np(_run(case, x))
    y_ref = oracle.gemm(xb, case.Wd)
    assert norm_err(full, y_ref, xb, case.Wd) <= TOL
    for B in (1, 4, 5, 8, 9):
        y = _np(_run(case, x[:B]))
        assert np.array_equal(y, full[:B]), "width %d differs from 16" % B


@pytest.fixture(scope="module")
def nvfp4_ffn():
    return (Case("nvfp4", INTER, HIDDEN, seed=inputs.W_SEED),
            Case("nvfp4", INTER, HIDDEN, seed=inputs.W2_SEED),
            Case("nvfp4", HIDDEN, INTER, seed=inputs.W3_SEED))


@pytest.mark.parametrize("M", [2048, 7235])
def test_nvfp4_prefill_ffn_chain(nvfp4_ffn, M):
    cg, cu, cd = nvfp4_ffn
    x = inputs.activations(M, HIDDEN, seed=inputs.X_SEED).cuda()
    h = qgemm.ffn_gate_up(x, cg.pw, cu.pw)
    y = _np(qgemm.run(h, cd.pw))
    torch.cuda.synchronize()
    rows = inputs.sample_rows(M)
    xb = inputs.bf16_bits(x.cpu())[rows]
    g, u, h_ref = oracle.ffn_gate_up(xb, cg.Wd, cu.Wd)
    h_gpu = bf16_bits_of(h)[rows]
    bad, worst = h_bound_violations(h_gpu, g, u, xb, cg.Wd, cu.Wd)
    assert bad == 0, "h: %d outputs outside the bound (worst ratio %.3g)" % (bad, worst)
    # down projection: y_gpu = GEMM(h_gpu), y_ref = exact(h_ref).  Per output,
    # |y_gpu - y_ref| <= TOL ||h_gpu|| ||w|| + ||h_gpu - h_ref|| ||w||  (GEMM bound, Cauchy-Schwarz)
    hg = oracle.bf16_decode_array(h_gpu)
    hr = oracle.bf16_decode_array(h_ref)
    y_ref = oracle.gemm(h_ref, cd.Wd)
    wn = np.sqrt((cd.Wd ** 2).sum(axis=1))[None, :]
    bound = (TOL * np.sqrt((hg ** 2).sum(axis=1))[:, None]
             + np.sqrt(((hg - hr) ** 2).sum(axis=1))[:, None]) * wn
    assert np.all(np.abs(y[rows] - y_ref) <= bound)
    # the down projection on the oracle's own h at the plain bar: the sampled rows of the
    # GPU's h are replaced by h_ref, and the full M-row GEMM runs in the same launch
    # configuration (rows are independent, so the others do not affect the sampled ones)
    h_mix = h.clone()
    h_mix[torch.from_numpy(rows).cuda()] = inputs.bits_to_bf16(h_ref).cuda()
    y_mix = _np(qgemm.run(h_mix, cd.pw))
    torch.cuda.synchronize()
    err = norm_err(y_mix[rows], y_ref, h_ref, cd.Wd)
    assert err <= TOL, "down projection on h_ref: normalised error %.3e" % err


def test_mxfp4_serving_mix():
    for N, K, seed in ((INTER, HIDDEN, inputs.W_SEED), (HIDDEN, INTER, inputs.W3_SEED)):
        case = Case("mxfp4", N, K, seed=seed)
        x = inputs.activations(32, K, seed=inputs.X_SEED).cuda()
        xb = inputs.bf16_bits(x.cpu())
        y = _np(_run(case, x))
        assert norm_err(y, oracle.gemm(xb, case.Wd), xb, case.Wd) <= TOL
        xp = inputs.activations(8192, K, seed=inputs.X_SEED + 100).cuda()
        yp = _np(_run(case, xp))
        rows = inputs.sample_rows(8192)
        _check_rows(case, yp, inputs.bf16_bits(xp.cpu()), rows)
        del case


def test_fp8_27b_widths_and_prefill():
    """FP8 (E4M3, per-tensor scale) at the 27B shapes: the batch-8 verify widths and decode
    widths on the gate/up shape, bitwise invariant; the down shape at B = 64; and an M = 2048
    prefill chunk on sampled rows.  The device packer gives the oracle's bytes at full size."""
    case = Case("fp8", INTER, HIDDEN, seed=inputs.W_SEED)
    pw = qgemm.pack("fp8", torch.from_numpy(case.W).cuda())
    torch.cuda.synchronize()
    ct, _ = tile_packed("fp8", case.codes, case.scales, INTER, HIDDEN)
    assert np.array_equal(pw.codes.cpu().numpy(), ct)
    assert pw.tensor_scale.item() == case.ts
    del pw
    x = inputs.activations(64, HIDDEN, seed=inputs.X_SEED).cuda()
    xb = inputs.bf16_bits(x.cpu())
    full = _np(_run(case, x))
    _check_rows(case, full, xb, list(range(64)))
    for B in (1, 8, 9, 16):
        assert np.array_equal(_np(_run(case, x[:B])), full[:B]), "width %d differs from 64" % B
    xp = inputs.activations(2048, HIDDEN, seed=inputs.X_SEED + 100).cuda()
    _check_rows(case, _np(_run(case, xp)), inputs.bf16_bits(xp.cpu()), inputs.sample_rows(2048))
    del case
    down = Case("fp8", HIDDEN, INTER, seed=inputs.W3_SEED)
    xd = inputs.activations(64, INTER, seed=inputs.X_SEED + 1).cuda()
    _check_rows(down, _np(_run(down, xd)), inputs.bf16_bits(xd.cpu()), [0, 31, 63])


@pytest.mark.parametrize("fmt", ["q8_0", "nvfp4", "fp8"])
def test_ffn_gate_up_decode_widths_27b(fmt):
    """The fused gate+up at the 27B gate/up shape and decode widths: every unit holds many
    A-slot groups, so both MMA issuers alternate through the A ring many times."""
    cg = Case(fmt, INTER, HIDDEN, seed=inputs.W_SEED)
    cu = Case(fmt, INTER, HIDDEN, seed=inputs.W2_SEED)
    x = inputs.activations(65, HIDDEN, seed=inputs.X_SEED).cuda()
    full = bf16_bits_of(qgemm.ffn_gate_up(x, cg.pw, cu.pw))
    torch.cuda.synchronize()
    assert qgemm.device_status(reset=False) == qgemm.OK
    rows = [0, 1, 15, 16, 63, 64]
    xb = inputs.bf16_bits(x.cpu())[rows]
    g, u, _ = oracle.ffn_gate_up(xb, cg.Wd, cu.Wd)
    bad, worst = h_bound_violations(full[rows], g, u, xb, cg.Wd, cu.Wd)
    assert bad == 0, "%d outputs outside the bound (worst ratio %.3g)" % (bad, worst)
    for M in (1, 16, 64):
        h = bf16_bits_of(qgemm.ffn_gate_up(x[:M], cg.pw, cu.pw))
        assert np.array_equal(h, full[:M]), "width %d differs from width 65" % M
