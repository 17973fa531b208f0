"""GPU parity of the beta-folded activation quantizer (dq_act_quant) against the oracle.

Bar: codes, group scales and the NVFP4 tensor scale bit-exact.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from calibration_free_weight_dualquant_b200 import binding, synth
from gpu_helpers import block_scale_values

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    binding.load_library()


def run_both(X: torch.Tensor, b: torch.Tensor, fmt: str, group: int, label: str):
    gpu = binding.dq_act_quant(X.cuda(), b.cuda(), fmt, group)
    Xin, xdt = synth.to_oracle_input(X)
    orc = oracle.act_quant(Xin, xdt, b.to(torch.float64).numpy(), fmt, group)
    a = block_scale_values(fmt, gpu["block_scales"])
    bad = np.argwhere(a != orc["a"])
    assert bad.size == 0, "%s scales differ at %d, first %s" % (label, len(bad), bad[:3].tolist())
    if fmt == "nvfp4":
        assert float(gpu["tensor_scale"].cpu()[0]) == orc["sT"], label
    codes = gpu["codes"].cpu().numpy()
    bad = np.argwhere(codes != orc["codes"])
    assert bad.size == 0, "%s codes differ at %d bytes, first %s" % (label, len(bad), bad[:3].tolist())
    return gpu, orc


_FMTS = [("nvfp4", 16), ("mxint4", 32), ("mxfp4", 32), ("int4", 8), ("int4", 16), ("int4", 32), ("int4", 64),
         ("int4", 128), ("int4", 256)]
_SHAPES = [
    (1, 256, torch.bfloat16, torch.bfloat16),
    (37, 4096, torch.bfloat16, torch.bfloat16),
    (129, 1536 + 256, torch.float16, torch.bfloat16),
    (64, 768, torch.bfloat16, torch.float16),
    (5, 1152, torch.bfloat16, torch.bfloat16),      # rows not a multiple of an item's rows; a partial slab
    (1030, 1152, torch.float16, torch.float16),     # warp ranges that cross slab boundaries
    (3, 1024 + 64, torch.bfloat16, torch.bfloat16),  # one lane-group past the last whole slab
    (2, 32768, torch.bfloat16, torch.bfloat16),     # more slabs than warps: a warp changes slab between items
]


@pytest.mark.parametrize("fmt,group,tokens,cols,xdt,bdt",
                         [f + s for f in _FMTS for s in _SHAPES if s[1] % f[1] == 0])
def test_act_parity(fmt, group, tokens, cols, xdt, bdt):
    X = synth.make_activations(tokens, cols, seed=tokens * 31 + cols).to(xdt)
    b = synth.make_col_scales(cols, seed=cols).to(bdt)
    run_both(X, b, fmt, group, "act")


@pytest.mark.parametrize("fmt,group,tokens,cols", [("nvfp4", 16, 8192, 4096), ("mxint4", 32, 8192, 14336),
                                                     ("int4", 64, 8192, 4096)])
def test_act_full_size(fmt, group, tokens, cols):
    """The prefill batches that the benchmark times (same shapes, seeds and launch), every output checked."""
    X = synth.make_activations(tokens, cols, seed=77)
    b = synth.make_col_scales(cols, seed=78)
    run_both(X, b, fmt, group, "full-size act")


@pytest.mark.parametrize("fmt", ["nvfp4", "mxint4", "int4", "mxfp4"])
def test_act_with_unit_scales_is_the_solvers_rtn(fmt):
    """With b = 1 the activation quantizer is the solver's RTN initial iterate (dq_rtn)."""
    X = synth.make_activations(96, 1024, seed=5).cuda()
    ones = torch.ones(1024, dtype=torch.bfloat16, device="cuda")
    g = binding.DEFAULT_GROUP[binding._fmt(fmt)]
    act = binding.dq_act_quant(X, ones, fmt, g)
    rtn = binding.dq_rtn(X, fmt, g)
    assert torch.equal(act["codes"], rtn["codes"])
    assert torch.equal(act["block_scales"], rtn["block_scales"])
    if fmt == "nvfp4":
        assert torch.equal(act["tensor_scale"], rtn["tensor_scale"])


def test_act_zeros_and_nonfinite():
    X = torch.zeros(8, 512, dtype=torch.bfloat16)
    X[3, 17:40] = 0.125
    b = synth.make_col_scales(512, seed=1)
    gpu, _ = run_both(X, b, "nvfp4", 16, "zeros")
    assert bool((gpu["codes"][0] == 0).all())
    Xn = X.clone().cuda()
    Xn[5, 100] = float("nan")
    for fmt, g in (("nvfp4", 16), ("mxint4", 32), ("int4", 64), ("mxfp4", 32)):
        with pytest.raises(binding.DQError) as e:
            binding.dq_act_quant(Xn, b.cuda(), fmt, g)
        assert e.value.status == 4, fmt


def test_act_argument_checks():
    lib = binding.load_library()
    X = synth.make_activations(4, 64, seed=2).cuda()
    b = torch.ones(64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.DQError) as e:
        binding.dq_act_quant(X, b, "mxint4", 16)
    assert e.value.status == 2
    with pytest.raises(binding.DQError) as e:
        binding.dq_act_quant(X[:, :48].contiguous(), b[:48], "int4", 32)  # 48 columns: not a multiple of 32
    assert e.value.status == 1
    assert lib.dq_act_quant(X.float().data_ptr(), 0, 4, 64, b.data_ptr(), 1, 2, 16, None, None, 0, None) != 0
