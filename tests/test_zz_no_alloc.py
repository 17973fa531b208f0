"""dq_solve_static: the solver for callers that cannot allocate device memory.

Such callers (a plugin whose host application owns all device memory, or a
path where an allocation would synchronise the device) pass only W and their
output buffers; the scratch is the library's own fixed device array.  These
tests call the entry point through the C ABI with preallocated buffers and
check it against dq_solve, which takes a caller workspace, on consecutive
calls that share that array.  This file is collected last on purpose.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from calibration_free_weight_dualquant_b200 import binding, synth
from gpu_helpers import block_scale_values, col_scale_values

pytestmark = pytest.mark.gpu

MSE_RTOL = 1e-4
DQ_EWORKSPACE = 3
DQ_ENONFINITE = 4
STATIC_SCRATCH_BYTES = 8 << 20


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    return binding.load_library()


def static_call(lib, W, fmt, group, iters, col_dtype):
    """dq_solve_static with every buffer allocated beforehand by the caller."""
    f = binding._fmt(fmt)
    rows, cols = W.shape
    out = binding.alloc_outputs(rows, cols, f, group, col_dtype, iters, W.device)
    out["mse"].fill_(-1.0)
    status = torch.full((1,), -1, dtype=torch.int32, device=W.device)
    o = binding._outputs_struct(out)
    torch.cuda.synchronize()
    st = lib.dq_solve_static(W.data_ptr(), binding._DTYPES[W.dtype], rows, cols, int(f), group, iters,
                             2 if col_dtype == "f16" else 1, ctypes.byref(o), status.data_ptr(),
                             torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return st, int(status.cpu()[0]), out


def assert_same(fmt, got, ref, label):
    assert torch.equal(got["codes"], ref["codes"]), label + " codes"
    np.testing.assert_array_equal(block_scale_values(fmt, got["block_scales"]),
                                  block_scale_values(fmt, ref["block_scales"]), err_msg=label + " block scales")
    np.testing.assert_array_equal(col_scale_values(got["col_scales"]), col_scale_values(ref["col_scales"]),
                                  err_msg=label + " col scales")
    if fmt == "nvfp4":
        assert float(got["tensor_scale"].cpu()[0]) == float(ref["tensor_scale"].cpu()[0]), label + " s_T"
    np.testing.assert_allclose(got["mse"].cpu().numpy(), ref["mse"].cpu().numpy(), rtol=MSE_RTOL, atol=0,
                               err_msg=label + " mse")


# Two calls in a row on the shared scratch: a larger NVFP4 solve, then a
# smaller INT4 one (stale partials or counters of the first would corrupt the
# second), then the first again.
CASES = [
    ("nvfp4", 16, "bf16", 1203, 800, 4, 11),
    ("int4", 64, "f16", 333, 704, 5, 12),
    ("nvfp4", 16, "bf16", 1203, 800, 4, 11),
]


def test_static_matches_workspace_entry_on_consecutive_calls(lib):
    wl = synth.WORKLOADS["nvfp4_g16_gateup_14336x4096"]
    for i, (fmt, group, cd, M, N, iters, seed) in enumerate(CASES):
        W = synth.make_weight(wl, M, N, seed=seed).cuda()
        assert binding.workspace_bytes(M, N, fmt, group) <= STATIC_SCRATCH_BYTES
        st, dev_st, got = static_call(lib, W, fmt, group, iters, cd)
        assert st == 0 and dev_st == 0, (st, dev_st)
        ref = binding.dq_solve(W, fmt, group, iters, cd)
        assert_same(fmt, got, ref, "call %d" % i)


def test_static_call_leaves_free_device_memory_unchanged(lib):
    """The call allocates nothing: the device's free memory (cudaMemGetInfo) is the same before and
    after a solve, once the library's device code is loaded (the first call on a device loads it).
    Every buffer the call touches is allocated beforehand; any device allocation inside the call
    would lower the free memory by at least one 2 MiB page."""
    wl = synth.WORKLOADS["nvfp4_g16_gateup_14336x4096"]
    fmt, group, cd, M, N, iters, seed = CASES[0]
    W = synth.make_weight(wl, M, N, seed=seed).cuda()
    out = binding.alloc_outputs(M, N, binding._fmt(fmt), group, cd, iters, W.device)
    status = torch.full((1,), -1, dtype=torch.int32, device=W.device)
    o = binding._outputs_struct(out)
    stream = torch.cuda.current_stream().cuda_stream

    def call():
        return lib.dq_solve_static(W.data_ptr(), binding._DTYPES[W.dtype], M, N, int(binding._fmt(fmt)), group,
                                   iters, 1, ctypes.byref(o), status.data_ptr(), stream)

    assert call() == 0  # loads the device code on this device if no call did yet
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert call() == 0
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert int(status.cpu()[0]) == 0
    assert free_after == free_before, (free_before, free_after)


def test_static_rejects_shape_beyond_scratch(lib):
    # one row of 2^20 columns needs about 16 MiB of scratch on a 148-SM GPU
    rows, cols, group = 1, 1 << 20, 64
    need = binding.workspace_bytes(rows, cols, "int4", group)
    assert need > STATIC_SCRATCH_BYTES
    W = torch.zeros(rows, cols, dtype=torch.float32, device="cuda")
    st, dev_st, out = static_call(lib, W, "int4", group, 1, "f16")
    assert st == DQ_EWORKSPACE
    assert dev_st == -1  # nothing was enqueued
    assert bool((out["mse"] == -1.0).all())


def test_static_reports_nonfinite_then_recovers(lib):
    W = torch.randn(64, 256, device="cuda") * 0.02
    W[3, 17] = float("nan")
    st, dev_st, _ = static_call(lib, W, "int4", 64, 2, "f16")
    assert st == 0 and dev_st == DQ_ENONFINITE
    W[3, 17] = 0.01
    st, dev_st, got = static_call(lib, W, "int4", 64, 2, "f16")
    assert st == 0 and dev_st == 0
    assert_same("int4", got, binding.dq_solve(W, "int4", 64, 2, "f16"), "after non-finite")
