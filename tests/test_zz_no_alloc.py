"""The allocation-free entry point, qgemm_run_noalloc.

Some callers cannot allocate device memory -- a serving runtime whose pool has already
reserved the GPU, a plugin that is only handed its input and output buffers -- so they cannot
provide the workspace qgemm_run asks for.  qgemm_run_noalloc runs the same kernels on a fixed
scratch array held inside the library.  These tests call it through the C ABI and check that
it gives bit for bit what qgemm_run gives (the same kernels with the same K split run on the
same inputs), and the oracle's result within the method's bound, on two calls in a row (the
second call finds the first call's data in the shared scratch), and that shapes too large for
the scratch are refused.

The file name sorts last so that pytest collects it after every other test; it must pass both
that way and alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from block_quantized_weight_qgemm_b200 import build as qbuild
from block_quantized_weight_qgemm_b200 import inputs
from block_quantized_weight_qgemm_b200 import qgemm
from gpu_helpers import TOL, Case, norm_err

SCRATCH_BYTES = 32 << 20  # QGEMM_NOALLOC_SCRATCH_BYTES in include/qgemm.h


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return qgemm.lib()


def _vp(t):
    return ctypes.c_void_p(t.data_ptr())


def test_oversize_shape_is_refused_before_device_work(lib):
    # needs no GPU: the size check comes before any device call
    fmt, N, K, B = 0, 8192, 65536, 256  # the f16 copy of x alone is 32 MiB
    need = qgemm.workspace_size("q8_0", N, K, B)
    assert need > SCRATCH_BYTES
    st = lib.qgemm_run_noalloc(fmt, 256, B, K, 256, 256, None, N, 256, 0, None)
    assert qgemm.STATUS[st] == "QGEMM_ERR_WORKSPACE"
    # argument checks match qgemm_run's
    assert lib.qgemm_run_noalloc(0, None, 4, 64, None, None, None, 8, None, 0, None) == 4
    assert lib.qgemm_run_noalloc(0, 16, 4, 64, 16, 16, None, 8, 16, 7, None) == 1
    assert lib.qgemm_run_noalloc(0, 8, 4, 64, 16, 16, None, 8, 16, 0, None) == 5


@pytest.mark.gpu
def test_noalloc_matches_qgemm_run_on_two_calls(lib):
    # two different problems, back to back on one stream; each needs split-K partials and the
    # f16 copy of x in the scratch, so the second call overwrites what the first left there
    cases = [("q8_0", 640, 2048, 5, torch.float32), ("nvfp4", 520, 4096, 37, torch.bfloat16)]
    stream = torch.cuda.current_stream()
    outs = []
    for fmt, N, K, B, ydt in cases:
        assert 0 < qgemm.workspace_size(fmt, N, K, B) <= SCRATCH_BYTES
        case = Case(fmt, N, K)
        x = inputs.activations(B, K, seed=inputs.X_SEED + B).cuda()
        y_ref = qgemm.run(x, case.pw, y_dtype=ydt)
        y = torch.full((B, N), float("nan"), dtype=ydt, device="cuda")
        pw = case.pw
        st = lib.qgemm_run_noalloc(qgemm.FORMATS[fmt], _vp(x), B, K, _vp(pw.codes),
                                   _vp(pw.scales),
                                   _vp(pw.tensor_scale) if pw.tensor_scale is not None else None,
                                   N, _vp(y), 1 if ydt == torch.bfloat16 else 0,
                                   ctypes.c_void_p(stream.cuda_stream))
        assert st == 0, lib.qgemm_status_str(st)
        outs.append((case, x, y, y_ref))
    torch.cuda.synchronize()
    assert qgemm.device_status() == 0
    for case, x, y, y_ref in outs:
        a = y.float().cpu().numpy().astype(np.float64)
        b = y_ref.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(a).all()
        # bit for bit what qgemm_run gives (NaN-filled y: every element was written)
        assert np.array_equal(a, b)
        xb = inputs.bf16_bits(x.cpu())
        err = norm_err(a, oracle.gemm(xb, case.Wd), xb, case.Wd)
        assert err <= TOL, err
