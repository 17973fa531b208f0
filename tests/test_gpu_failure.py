"""Failure detection on the GPU without a fault: every wait of the per-iteration kernel is bounded in
time, gives up with a status the host reads, and leaves the context usable.

The self-test entry point runs one of the kernel's waits on something that nothing releases: a pending
count in global memory that nothing counts down (the wait for a block-column's exactly updated column
scales), or a shared-memory ring barrier that no copy completes and nobody arrives at (the tile
pipeline's wait).  No copy is issued and no GPU fault, trap or hang is involved.
"""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

import oracle
from calibration_free_weight_dualquant_b200 import binding, synth

DQ_ECUDA = 5


@pytest.mark.gpu
@pytest.mark.parametrize("which", [0, 1])
def test_bounded_wait_gives_up_with_a_status_and_the_context_stays_usable(which):
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    st = binding.wait_selftest(ws, which)
    elapsed = time.time() - t0
    assert st == DQ_ECUDA
    assert 0.5 < elapsed < 60.0, elapsed  # about the 1 s limit of a wait
    # the same context solves correctly afterwards
    wl = synth.WORKLOADS["nvfp4_g16_gateup_14336x4096"]
    W = synth.make_weight(wl, 64, 512, seed=21)
    gpu = binding.dq_solve(W.cuda(), "nvfp4", 16, 3, "bf16")
    Win, wdt = synth.to_oracle_input(W)
    orc = oracle.solve(Win, wdt, "nvfp4", 16, 3, "bf16")
    assert np.array_equal(gpu["codes"].cpu().numpy(), orc["codes"])


@pytest.mark.gpu
def test_wait_selftest_rejects_bad_arguments():
    small = torch.empty(128, dtype=torch.uint8, device="cuda")
    with pytest.raises(binding.DQError) as e:
        binding.wait_selftest(small)
    assert e.value.status == 3  # DQ_EWORKSPACE
