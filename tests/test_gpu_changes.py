"""GPU parity of the changed-code counts (dq_options.code_changes) against the oracle.

code_changes[t] = elements whose code differs between the iterates after
iterations t-1 and t (DualQuant summary §4.3, App. B: the quantized matrix
stabilizes).  Bar: every count equal to the oracle's, and a counting solve
returns exactly what the same solve without counting returns.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from calibration_free_weight_dualquant_b200 import binding, synth
from gpu_helpers import compare_with_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    binding.load_library()


def _same(a: dict, b: dict):
    for k in ("codes", "block_scales", "col_scales", "tensor_scale", "mse"):
        assert torch.equal(a[k], b[k]), k


@pytest.mark.parametrize("mode,init", [("dual", "rtn"), ("dual", "l1"), ("row", "rtn"), ("col", "l1")])
@pytest.mark.parametrize("fmt,group,col_dtype", [("nvfp4", 16, "bf16"), ("mxint4", 32, "bf16"), ("int4", 64, "f16"),
                                              ("mxfp4", 32, "bf16"), ("int4", 128, "bf16"),
                                              ("mxint8", 32, "bf16"), ("mxfp8", 32, "bf16")])
@pytest.mark.parametrize("rows,cols,dtype,iters", [(97, 768 + 128, torch.bfloat16, 6), (64, 512, torch.float32, 4),
                                                  (40, 256, torch.float16, 1)])
def test_changes_match_oracle(mode, init, fmt, group, col_dtype, rows, cols, dtype, iters):
    if cols % group:
        pytest.skip("cols not a multiple of the group")
    wl = synth.WORKLOADS["nvfp4_g16_gateup_14336x4096"]
    W = synth.make_weight(wl, rows, cols, seed=rows + cols).to(dtype)
    gpu = binding.dq_solve(W.cuda(), fmt, group, iters, col_dtype, mode=mode, init=init, changes=True)
    plain = binding.dq_solve(W.cuda(), fmt, group, iters, col_dtype, mode=mode, init=init)
    _same(gpu, plain)
    Win, wdt = synth.to_oracle_input(W)
    orc = oracle.solve(Win, wdt, fmt, group, iters, col_dtype, mode=mode, init=init, changes=True)
    compare_with_oracle(fmt, gpu, orc, 1e-4, "changes")
    got = gpu["code_changes"].cpu().numpy()
    np.testing.assert_array_equal(got, orc["changes"].astype(np.int64))
    assert got[0] == 0


def test_changes_zero_iterations_and_warm_start():
    wl = synth.WORKLOADS["mxint4_g32_downproj_4096x14336"]
    W = synth.make_weight(wl, 64, 512, seed=2).cuda()
    z = binding.dq_solve(W, "mxint4", 32, 0, "bf16", changes=True)
    assert z["code_changes"].cpu().tolist() == [0]
    full = binding.dq_solve(W, "mxint4", 32, 8, "bf16", changes=True)
    first = binding.dq_solve(W, "mxint4", 32, 3, "bf16")
    warm = binding.dq_solve(W, "mxint4", 32, 5, "bf16", init="given", changes=True,
                            init_scales={k: first[k] for k in ("block_scales", "col_scales", "tensor_scale")})
    assert torch.equal(full["code_changes"][4:], warm["code_changes"][1:])


def test_changes_full_size():
    """MXINT4 4096x14336, 20 iterations: every count equal to the oracle's."""
    wl = synth.WORKLOADS["mxint4_g32_downproj_4096x14336"]
    W = synth.make_weight(wl, wl.rows, wl.cols, seed=wl.seed)
    gpu = binding.dq_solve(W.cuda(), wl.fmt, wl.group, wl.iters, wl.col_dtype, changes=True)
    Win, wdt = synth.to_oracle_input(W)
    orc = oracle.solve(Win, wdt, wl.fmt, wl.group, wl.iters, wl.col_dtype, changes=True)
    np.testing.assert_array_equal(gpu["code_changes"].cpu().numpy(), orc["changes"].astype(np.int64))
    compare_with_oracle(wl.fmt, gpu, orc, 1e-4, wl.name)
