"""Routed mixture-of-experts variants -- qgemm_moe_run (routed down projection) and
qgemm_moe_gate_up (routed fused gate+up with the SiLU(g)*u epilogue) -- against the oracle:
each expert's rows through the oracle's GEMM or fused FFN with that expert's dequantised
weights (Atlas issue, the routed expert kernels of the "Per-32-K-step hot loop" table; Strix
Halo prefill journey, the fused gate/up + SwiGLU for the MoE and the routed down
projections).  Experts with no rows, a ragged last row tile and the wide (bf16-operand) path
are covered; a row's output must not depend on the other experts' rows or on max_rows."""
import numpy as np
import pytest
import torch

import oracle
from block_quantized_weight_qgemm_b200 import inputs
from block_quantized_weight_qgemm_b200 import qgemm
from gpu_helpers import TOL, Case, bf16_bits_of, h_bound_violations, norm_err

pytestmark = pytest.mark.gpu

FMTS = ["q8_0", "nvfp4", "mxfp4", "fp8"]
COUNTS = [0, 5, 17, 1, 0, 64, 3, 9]  # rows per expert, empty experts included
N, K = 300, 512                      # two full 128-row tiles and a ragged tail


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_quantized_weight_qgemm_b200 import build
    build.build()
    qgemm.lib()
    qgemm.device_status(reset=True)
    yield
    assert qgemm.device_status(reset=True) == qgemm.OK


def _offsets(counts):
    return torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)).cuda()


@pytest.fixture(scope="module")
def experts():
    out = {}
    for fmt in FMTS:
        E = len(COUNTS)
        out[fmt] = {name: [Case(fmt, N, K, seed=100 * i + j) for i in range(E)]
                    for j, name in enumerate(("gate", "up", "down"))}
    return out


def _table(cases):
    return qgemm.ExpertTable([c.pw for c in cases])


@pytest.mark.parametrize("fmt", FMTS)
def test_moe_run_matches_oracle_per_expert(experts, fmt):
    cs = experts[fmt]["down"]
    M = sum(COUNTS)
    x = inputs.activations(M, K, seed=31).cuda()
    xb = inputs.bf16_bits(x.cpu())
    off = _offsets(COUNTS)
    y = qgemm.moe_run(x, off, _table(cs), max_rows=max(COUNTS))
    torch.cuda.synchronize()
    y = y.double().cpu().numpy()
    o = off.cpu().numpy()
    for e, c in enumerate(cs):
        rows = slice(int(o[e]), int(o[e + 1]))
        if o[e + 1] == o[e]:
            continue
        err = norm_err(y[rows], oracle.gemm(xb[rows], c.Wd), xb[rows], c.Wd)
        assert err <= TOL, (e, err)
    # bf16 output is the fp32 result rounded once
    yb = qgemm.moe_run(x, off, _table(cs), max_rows=max(COUNTS), y_dtype=torch.bfloat16)
    assert np.array_equal(yb.double().cpu().numpy(),
                          torch.from_numpy(y).to(torch.bfloat16).double().numpy())


@pytest.mark.parametrize("fmt", FMTS)
def test_moe_gate_up_matches_oracle_per_expert(experts, fmt):
    gs, us = experts[fmt]["gate"], experts[fmt]["up"]
    M = sum(COUNTS)
    x = inputs.activations(M, K, seed=32).cuda()
    xb = inputs.bf16_bits(x.cpu())
    off = _offsets(COUNTS)
    h = bf16_bits_of(qgemm.moe_gate_up(x, off, _table(gs), _table(us), max_rows=max(COUNTS)))
    o = off.cpu().numpy()
    for e in range(len(COUNTS)):
        rows = slice(int(o[e]), int(o[e + 1]))
        if o[e + 1] == o[e]:
            continue
        g, u, _ = oracle.ffn_gate_up(xb[rows], gs[e].Wd, us[e].Wd)
        bad, worst = h_bound_violations(h[rows], g, u, xb[rows], gs[e].Wd, us[e].Wd)
        assert bad == 0, (e, bad, worst)


@pytest.mark.parametrize("fmt", ["q8_0", "nvfp4"])
def test_moe_rows_independent_of_routing_and_max_rows(experts, fmt):
    # expert 5's 64 rows: alone, among the others, with other max_rows, and every prefix width
    gs, us, ds = experts[fmt]["gate"], experts[fmt]["up"], experts[fmt]["down"]
    M = sum(COUNTS)
    x = inputs.activations(M, K, seed=33).cuda()
    off = _offsets(COUNTS)
    full_y = qgemm.moe_run(x, off, _table(ds), max_rows=64).cpu()
    full_h = qgemm.moe_gate_up(x, off, _table(gs), _table(us), max_rows=64).cpu()
    o = off.cpu().numpy()
    r0, r1 = int(o[5]), int(o[6])
    for mr in (64, 100, 256):
        assert torch.equal(qgemm.moe_run(x, off, _table(ds), max_rows=mr).cpu(), full_y)
    alone = [0] * len(COUNTS)
    for w in (1, 7, 16, 17, 63, 64):
        alone[5] = w
        xa = x[r0:r0 + w].contiguous()
        ya = qgemm.moe_run(xa, _offsets(alone), _table(ds), max_rows=w).cpu()
        ha = qgemm.moe_gate_up(xa, _offsets(alone), _table(gs), _table(us), max_rows=w).cpu()
        assert torch.equal(ya, full_y[r0:r0 + w]), w
        assert torch.equal(ha, full_h[r0:r0 + w]), w


@pytest.mark.parametrize("fmt", ["nvfp4", "q8_0"])
def test_moe_wide_expert_bf16_path(experts, fmt):
    # one expert above 256 rows takes the bf16-operand path; parity per expert
    counts = [0, 300, 2, 0, 0, 0, 0, 0]
    gs, us, ds = experts[fmt]["gate"], experts[fmt]["up"], experts[fmt]["down"]
    M = sum(counts)
    x = inputs.activations(M, K, seed=34).cuda()
    xb = inputs.bf16_bits(x.cpu())
    off = _offsets(counts)
    y = qgemm.moe_run(x, off, _table(ds), max_rows=300).double().cpu().numpy()
    h = bf16_bits_of(qgemm.moe_gate_up(x, off, _table(gs), _table(us), max_rows=300))
    for e, (a, b) in ((1, (0, 300)), (2, (300, 302))):
        rows = slice(a, b)
        assert norm_err(y[rows], oracle.gemm(xb[rows], ds[e].Wd), xb[rows], ds[e].Wd) <= TOL
        g, u, _ = oracle.ffn_gate_up(xb[rows], gs[e].Wd, us[e].Wd)
        assert h_bound_violations(h[rows], g, u, xb[rows], gs[e].Wd, us[e].Wd)[0] == 0


def test_moe_bad_table_entry_is_refused_on_the_device(experts):
    # a NULL and a misaligned expert pointer: the kernel checks its table entries before any
    # copy, skips those experts and reports QGEMM_ERR_DEVICE_ARG; the other experts are right
    cs = experts["nvfp4"]["down"]
    M = sum(COUNTS)
    x = inputs.activations(M, K, seed=35).cuda()
    xb = inputs.bf16_bits(x.cpu())
    off = _offsets(COUNTS)
    tab = _table(cs)
    tab.codes[1] = 0
    tab.codes[2] = tab.codes[2] + 8
    y = torch.full((M, N), 7.0, device="cuda")
    qgemm.moe_run(x, off, tab, max_rows=64, y=y)
    assert qgemm.device_status(reset=True) == 10  # QGEMM_ERR_DEVICE_ARG
    y = y.double().cpu().numpy()
    o = off.cpu().numpy()
    assert np.all(y[o[1]:o[3]] == 7.0)  # experts 1 and 2 untouched
    rows = slice(int(o[5]), int(o[6]))
    assert norm_err(y[rows], oracle.gemm(xb[rows], cs[5].Wd), xb[rows], cs[5].Wd) <= TOL


def test_moe_flash_next_expert_shapes():
    """Routed experts at the Flash-Next expert shape (hidden 2048, expert FFN 512; the pages
    give 512 experts with top-10 routing, this test routes 48 tokens top-10 over 32 of them),
    NVFP4: gate+up -> h and the down projection, every row of 8 experts against the oracle."""
    E, T, k, H, F = 32, 48, 10, 2048, 512
    tok, exp_, off_np = inputs.routing(T, E, k, seed=7)
    gs = [Case("nvfp4", F, H, seed=1000 + e) for e in range(E)]
    us = [Case("nvfp4", F, H, seed=2000 + e) for e in range(E)]
    ds = [Case("nvfp4", H, F, seed=3000 + e) for e in range(E)]
    xt = inputs.activations(T, H, seed=41)
    x = xt[torch.from_numpy(tok)].contiguous().cuda()     # routed rows, grouped by expert
    M = x.shape[0]
    off = torch.from_numpy(off_np).cuda()
    mr = int(np.diff(off_np).max())
    h = qgemm.moe_gate_up(x, off, _table(gs), _table(us), max_rows=mr)
    hin = inputs.activations(M, F, seed=42).cuda()          # an independent input for down
    y = qgemm.moe_run(hin, off, _table(ds), max_rows=mr).double().cpu().numpy()
    hb = bf16_bits_of(h)
    xb = inputs.bf16_bits(x.cpu())
    hinb = inputs.bf16_bits(hin.cpu())
    for e in range(0, E, 4):
        rows = slice(int(off_np[e]), int(off_np[e + 1]))
        if off_np[e + 1] == off_np[e]:
            continue
        g, u, _ = oracle.ffn_gate_up(xb[rows], gs[e].Wd, us[e].Wd)
        assert h_bound_violations(hb[rows], g, u, xb[rows], gs[e].Wd, us[e].Wd)[0] == 0, e
        assert norm_err(y[rows], oracle.gemm(hinb[rows], ds[e].Wd), hinb[rows], ds[e].Wd) <= TOL, e
