"""Batched solves through dq_solve_batched, and the 224-matrix Llama-3.1-8B linear set.

The whole set is 7.0 G elements; the oracle checks a subset of it (layer 0's
seven matrices and three seeded others) in both formats, every output of every
checked matrix bit-exact and every MSE entry within 1e-4 relative.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from calibration_free_weight_dualquant_b200 import binding, synth
from gpu_helpers import compare_with_oracle

pytestmark = pytest.mark.gpu

MSE_RTOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    binding.load_library()


def _same(a: dict, b: dict):
    for k in ("codes", "block_scales", "col_scales", "tensor_scale", "mse"):
        assert torch.equal(a[k], b[k]), k


@pytest.mark.parametrize("fmt,group,col_dtype", [("nvfp4", 16, "bf16"), ("mxint4", 32, "bf16"), ("int4", 64, "f16"),
                                              ("mxfp4", 32, "bf16"), ("mxint8", 32, "bf16"), ("mxfp8", 32, "bf16")])
def test_batched_equals_one_by_one(fmt, group, col_dtype):
    wl = synth.WORKLOADS["nvfp4_g16_gateup_14336x4096"]
    shapes = [(300, 512), (77, 1024), (513, 256), (1024, 768)]
    Ws = [synth.make_weight(wl, m, n, seed=40 + i).cuda() for i, (m, n) in enumerate(shapes)]
    Ws[2] = Ws[2].to(torch.float16)
    got = binding.dq_solve_batched(Ws, fmt, group, 5, col_dtype)
    for W, g in zip(Ws, got):
        _same(g, binding.dq_solve(W, fmt, group, 5, col_dtype))


def test_batched_status_per_matrix():
    wl = synth.WORKLOADS["nvfp4_g16_gateup_14336x4096"]
    Ws = [synth.make_weight(wl, 64, 256, seed=50 + i).cuda() for i in range(3)]
    Ws[1][5, 7] = float("inf")
    status = torch.full((3,), -1, dtype=torch.int32, device="cuda")
    outs = binding.dq_solve_batched(Ws, "nvfp4", 16, 3, "bf16", status=status, check=False)
    torch.cuda.synchronize()
    assert status.cpu().tolist() == [0, 4, 0]
    for i in (0, 2):  # the finite matrices are solved as if alone
        _same(outs[i], binding.dq_solve(Ws[i], "nvfp4", 16, 3, "bf16"))


def test_batched_rejects_before_enqueue():
    wl = synth.WORKLOADS["nvfp4_g16_gateup_14336x4096"]
    Ws = [synth.make_weight(wl, 64, 256, seed=60).cuda(), synth.make_weight(wl, 64, 264, seed=61).cuda()]
    outs = [binding.alloc_outputs(W.shape[0], W.shape[1], "nvfp4", 16 if i == 0 else 8, "bf16", 2, "cuda")
            for i, W in enumerate(Ws)]
    for o in outs:
        o["mse"].fill_(-1.0)
    with pytest.raises(binding.DQError) as e:
        binding.dq_solve_batched(Ws, "nvfp4", 16, 2, "bf16", outs=outs)  # 264 columns: not a multiple of 16
    assert e.value.status == 1 and "matrix 1" in str(e.value)
    torch.cuda.synchronize()
    assert bool((outs[0]["mse"] == -1.0).all())  # nothing was enqueued


def llama_subset():
    """Layer 0's seven matrices and three seeded others (layer, projection)."""
    rng = np.random.Generator(np.random.PCG64(2024))
    others = [(int(rng.integers(1, synth.LLAMA31_8B_LAYERS)), int(rng.integers(0, 7))) for _ in range(3)]
    return [(0, pid) for pid in range(7)] + others


@pytest.mark.parametrize("fmt", ["nvfp4", "mxint4"])
def test_llama_set_subset_against_oracle(fmt):
    wls = [synth.llama_set_workload(layer, pid, fmt) for layer, pid in llama_subset()]
    Ws = [synth.make_weight_device(wl, "cuda") for wl in wls]
    outs = binding.dq_solve_batched(Ws, fmt, wls[0].group, wls[0].iters, wls[0].col_dtype)
    for wl, W, gpu in zip(wls, Ws, outs):
        Win, wdt = synth.to_oracle_input(W.cpu())
        orc = oracle.solve(Win, wdt, fmt, wl.group, wl.iters, wl.col_dtype)
        compare_with_oracle(fmt, gpu, orc, MSE_RTOL, wl.name)
        del orc
