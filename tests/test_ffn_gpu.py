"""qgemm_ffn_gate_up on the GPU against the oracle: the fused gate+up GEMM with the
SiLU(g)*u epilogue (Atlas issue, "fused gate+up with dual accumulators").

h is bf16, so it is checked against the bound of gpu_helpers.h_bound_violations: one bf16
rounding of the exact h plus the first-order effect of the GEMM bound on g and u."""
import numpy as np
import pytest
import torch

import oracle
from block_quantized_weight_qgemm_b200 import inputs
from block_quantized_weight_qgemm_b200 import qgemm
from gpu_helpers import Case, bf16_bits_of, h_bound_violations

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


@pytest.fixture(scope="module")
def pairs():
    # 300 rows: two full 128-row tiles and a ragged tail; K = 1024 spans several stages
    return {f: (Case(f, 300, 1024, seed=21), Case(f, 300, 1024, seed=22)) for f in FMTS}


def _h(x, cg, cu):
    h = qgemm.ffn_gate_up(x.cuda().contiguous(), cg.pw, cu.pw)
    torch.cuda.synchronize()
    return bf16_bits_of(h)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 5, 64, 65, 129, 256, 257, 300])
def test_ffn_parity_small(pairs, fmt, M):
    cg, cu = pairs[fmt]
    x = inputs.activations(M, cg.K, seed=23)
    xb = inputs.bf16_bits(x)
    g, u, _ = oracle.ffn_gate_up(xb, cg.Wd, cu.Wd)
    h = _h(x, cg, cu)
    bad, worst = h_bound_violations(h, g, u, xb, cg.Wd, cu.Wd)
    assert bad == 0, "%d outputs outside the bound (worst ratio %.3g)" % (bad, worst)


@pytest.mark.parametrize("fmt", FMTS)
def test_ffn_matches_oracle_h_mostly_exactly(pairs, fmt):
    # where the exact h is not close to a bf16 rounding boundary both sides round alike.  The
    # Q8_0 weight operand is q*d rounded once to f16 (relative error up to 2^-12), so its g and
    # u sit further from the exact values and h's last rounding flips more often.
    cg, cu = pairs[fmt]
    x = inputs.activations(16, cg.K, seed=24)
    xb = inputs.bf16_bits(x)
    _, _, h_ref = oracle.ffn_gate_up(xb, cg.Wd, cu.Wd)
    h = _h(x, cg, cu)
    assert np.mean(h == h_ref) > (0.7 if fmt == "q8_0" else 0.97)


@pytest.mark.parametrize("fmt", FMTS)
def test_ffn_batch_invariance(pairs, fmt):
    cg, cu = pairs[fmt]
    x = inputs.activations(256, cg.K, seed=25)
    full = _h(x, cg, cu)
    for M in (1, 2, 7, 16, 63, 64, 65, 70, 76, 128, 129, 200, 255):
        assert np.array_equal(_h(x[:M], cg, cu), full[:M]), "width %d differs from width 256" % M
    for s0, M in [(3, 64), (100, 70)]:
        assert np.array_equal(_h(x[s0:s0 + M], cg, cu), full[s0:s0 + M]), (s0, M)


@pytest.mark.parametrize("fmt", FMTS)
def test_ffn_wide_chunks_parity_and_row_independence(pairs, fmt):
    # 4300 rows run as three balanced chunks (1440, 1440, 1420 rows) of two GEMMs and a SiLU
    # pass each; above 256 rows a row of h still depends only on its own row of x, so a
    # 300-row window across a chunk boundary (a single chunk when run alone) matches bitwise
    cg, cu = pairs[fmt]
    M = 4300
    x = inputs.activations(M, cg.K, seed=26)
    xb = inputs.bf16_bits(x)
    g, u, _ = oracle.ffn_gate_up(xb, cg.Wd, cu.Wd)
    h = _h(x, cg, cu)
    bad, worst = h_bound_violations(h, g, u, xb, cg.Wd, cu.Wd)
    assert bad == 0, "%d outputs outside the bound (worst ratio %.3g)" % (bad, worst)
    s0 = 1300
    assert np.array_equal(_h(x[s0:s0 + 300], cg, cu), h[s0:s0 + 300])
