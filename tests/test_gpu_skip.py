"""Block-columns at a fixed point: skipping them gives exactly the outputs of full passes.

A block-column (the rows x group slab under one column of blocks) holds its own block scales and
column scales, and one BCD iteration maps them to their next values from that slab alone
(reproduction README, "Core equations": the block update reads the block's elements and their column
scales, the column update reads the column and the block scales of its blocks; the NVFP4 tensor scale
is fixed at init).  A block-column whose scales come out of an iteration unchanged therefore repeats
the same iteration forever, and the solver skips it from then on.  These tests run each workload's
law and format with and without skipping and require identical codes, scales and changed-code counts,
bit for bit, and that skipping did skip work.  The per-iteration MSE is a sum of per-block-column
totals, each built from fp32 runs of 8 rows of a lane added into fp64; a skipped block-column keeps the
total of the pass that last computed it, whose CTA split of the rows (and so its grouping of rows into
runs) may differ from a full pass's, so the MSE may differ by the rounding of those runs (about 1e-9
relative): it is held to 1e-7 here, against the oracle to 1e-4 elsewhere.
"""
from __future__ import annotations

import pytest
import torch

from calibration_free_weight_dualquant_b200 import binding, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    binding.load_library()


def _same(a: dict, b: dict, keys=("codes", "block_scales", "col_scales", "tensor_scale")):
    for k in keys:
        assert torch.equal(a[k], b[k]), k
    torch.testing.assert_close(a["mse"], b["mse"], rtol=1e-7, atol=0)


NAMES = ["nvfp4_g16_gateup_14336x4096", "mxint4_g32_downproj_4096x14336", "int4_g64_qproj_4096x4096",
         "mxfp4_g32_downproj_4096x14336", "mxint8_g32_downproj_4096x14336", "mxfp8_g32_downproj_4096x14336"]


@pytest.mark.parametrize("name", NAMES)
@pytest.mark.parametrize("changes", [False, True])
def test_skipping_equals_full_passes(name, changes):
    wl = synth.WORKLOADS[name]
    rows, cols = 1536, min(wl.cols, 2048)
    W = synth.make_weight(wl, rows, cols, seed=wl.seed + 3).cuda()
    T = wl.iters
    skip = binding.dq_solve(W, wl.fmt, wl.group, T, wl.col_dtype, changes=changes)
    full = binding.dq_solve(W, wl.fmt, wl.group, T, wl.col_dtype, changes=changes, full_passes=True)
    _same(skip, full, ("codes", "block_scales", "col_scales", "tensor_scale") +
          (("code_changes",) if changes else ()))
    nb = cols // wl.group
    assert binding.active_block_columns(full["workspace"]) == T * nb
    n_skip = binding.active_block_columns(skip["workspace"])
    assert 0 < n_skip <= T * nb
    if wl.fmt == "nvfp4":  # the E4M3 and bf16 grids settle early on this law
        assert n_skip < T * nb


@pytest.mark.parametrize("mode", ["row", "col"])
def test_skipping_in_ablation_modes(mode):
    wl = synth.WORKLOADS["nvfp4_g16_gateup_14336x4096"]
    W = synth.make_weight(wl, 777, 1056, seed=31).cuda()
    skip = binding.dq_solve(W, "nvfp4", 16, 12, "bf16", mode=mode)
    full = binding.dq_solve(W, "nvfp4", 16, 12, "bf16", mode=mode, full_passes=True)
    _same(skip, full)
