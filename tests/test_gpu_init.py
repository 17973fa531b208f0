"""GPU parity of the init variants of dq_solve_ex against the oracle.

Per-column L1-norm init (DualQuant summary §5.3) and the warm start from given
scales.  Bar: codes, block and column scales and the NVFP4 tensor scale
bit-exact; every MSE entry within 1e-4 relative.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from calibration_free_weight_dualquant_b200 import binding, synth
from gpu_helpers import block_scale_values, col_scale_values, compare_with_oracle

pytestmark = pytest.mark.gpu

MSE_RTOL = 1e-4
FORMATS = [("nvfp4", 16, "bf16"), ("mxint4", 32, "bf16"), ("int4", 64, "f16"), ("mxfp4", 32, "bf16"),
           ("int4", 16, "bf16"), ("mxint8", 32, "bf16"), ("mxfp8", 32, "bf16")]
# one configuration per format
PRIMARY = [f for f in FORMATS if f != ("int4", 16, "bf16")]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    binding.load_library()


def weight(rows, cols, seed, dtype=torch.bfloat16, name="nvfp4_g16_gateup_14336x4096"):
    return synth.make_weight(synth.WORKLOADS[name], rows, cols, seed=seed).to(dtype)


def oracle_of(W: torch.Tensor, fmt, group, iters, col_dtype, **kw):
    Win, wdt = synth.to_oracle_input(W)
    return oracle.solve(Win, wdt, fmt, group, iters, col_dtype, **kw)


@pytest.mark.parametrize("fmt,group,col_dtype", FORMATS)
@pytest.mark.parametrize("rows,cols,dtype,iters", [
    (96, 512, torch.bfloat16, 0),
    (97, 768 + 64, torch.bfloat16, 6),      # ragged row tail, partial last strip
    (130, 1024, torch.float16, 4),
    (64, 256, torch.float32, 5),
])
def test_l1_init_parity(fmt, group, col_dtype, rows, cols, dtype, iters):
    if cols % group:
        pytest.skip("cols not a multiple of the group")
    W = weight(rows, cols, seed=rows * 7 + cols, dtype=dtype)
    gpu = binding.dq_solve(W.cuda(), fmt, group, iters, col_dtype, init="l1")
    orc = oracle_of(W, fmt, group, iters, col_dtype, init="l1")
    compare_with_oracle(fmt, gpu, orc, MSE_RTOL, "l1 %s %dx%d" % (fmt, rows, cols))
    assert not np.all(orc["b"] == 1.0)


@pytest.mark.parametrize("fmt,group,col_dtype", PRIMARY)
def test_l1_init_zero_columns_and_zero_matrix(fmt, group, col_dtype):
    W = weight(64, 512, seed=3)
    W[:, 17] = 0
    W[:, 300:340] = 0
    W[5, :] = 0
    gpu = binding.dq_solve(W.cuda(), fmt, group, 3, col_dtype, init="l1")
    orc = oracle_of(W, fmt, group, 3, col_dtype, init="l1")
    compare_with_oracle(fmt, gpu, orc, MSE_RTOL, "zeros")
    Z = torch.zeros(32, 256, dtype=torch.bfloat16)
    gz = binding.dq_solve(Z.cuda(), fmt, group, 2, col_dtype, init="l1")
    compare_with_oracle(fmt, gz, oracle_of(Z, fmt, group, 2, col_dtype, init="l1"), MSE_RTOL, "zero W")


def test_l1_init_extreme_magnitudes():
    """Column sums spanning the whole fp32 range: the exact sums keep every bit."""
    rng = np.random.Generator(np.random.PCG64(5))
    W = (rng.standard_normal((64, 256)) * np.exp2(rng.integers(-60, 60, (64, 256)))).astype(np.float32)
    W[:, 3] = np.float32(2.0 ** -140)     # a column of fp32 subnormals
    W[7, 9] = np.float32(3.0e38)          # one huge entry
    Wt = torch.from_numpy(W)
    for fmt, group, cd in (("int4", 64, "f16"), ("nvfp4", 16, "bf16"), ("mxint4", 32, "bf16")):
        gpu = binding.dq_solve(Wt.cuda(), fmt, group, 2, cd, init="l1")
        orc = oracle_of(Wt, fmt, group, 2, cd, init="l1")
        compare_with_oracle(fmt, gpu, orc, MSE_RTOL, "extreme " + fmt)


@pytest.mark.parametrize("fmt,group,col_dtype", PRIMARY)
def test_l1_init_full_size(fmt, group, col_dtype):
    """The init at the workload's full size: every scale and code of the initial iterate bit-exact."""
    name = {"nvfp4": "nvfp4_g16_gateup_14336x4096", "mxint4": "mxint4_g32_downproj_4096x14336",
            "int4": "int4_g64_qproj_4096x4096", "mxfp4": "mxfp4_g32_downproj_4096x14336",
            "mxint8": "mxint8_g32_downproj_4096x14336", "mxfp8": "mxfp8_g32_downproj_4096x14336"}[fmt]
    wl = synth.WORKLOADS[name]
    W = synth.make_weight(wl, wl.rows, wl.cols, seed=wl.seed)
    gpu = binding.dq_solve(W.cuda(), fmt, group, 0, col_dtype, init="l1")
    orc = oracle_of(W, fmt, group, 0, col_dtype, init="l1")
    compare_with_oracle(fmt, gpu, orc, MSE_RTOL, "full " + name)


def _given(gpu: dict) -> dict:
    return {k: gpu[k].clone() for k in ("block_scales", "col_scales", "tensor_scale")}


@pytest.mark.parametrize("init", ["rtn", "l1"])
@pytest.mark.parametrize("fmt,group,col_dtype", PRIMARY)
def test_warm_start_continues_the_iteration(init, fmt, group, col_dtype):
    """T1 iterations, then a warm start of T2 more, equal T1 + T2 iterations bit for bit; the oracle
    started from the same scales agrees."""
    W = weight(150, 768, seed=9).cuda()
    full = binding.dq_solve(W, fmt, group, 7, col_dtype, init=init)
    first = binding.dq_solve(W, fmt, group, 3, col_dtype, init=init)
    warm = binding.dq_solve(W, fmt, group, 4, col_dtype, init="given", init_scales=_given(first))
    for k in ("codes", "block_scales", "col_scales", "tensor_scale"):
        assert torch.equal(full[k], warm[k]), k
    assert torch.equal(full["mse"][3:], warm["mse"])
    orc = oracle_of(W.cpu(), fmt, group, 4, col_dtype, init="given",
                    a0=block_scale_values(fmt, first["block_scales"]), b0=col_scale_values(first["col_scales"]),
                    sT0=float(first["tensor_scale"].cpu()[0]))
    compare_with_oracle(fmt, warm, orc, MSE_RTOL, "warm " + fmt)


def test_warm_start_from_rtn_scales_is_rtn_init():
    W = weight(64, 512, seed=10).cuda()
    for fmt, group, cd in PRIMARY:
        r = binding.dq_solve(W, fmt, group, 3, cd)
        z = binding.dq_solve(W, fmt, group, 0, cd)
        g = binding.dq_solve(W, fmt, group, 3, cd, init="given", init_scales=_given(z))
        for k in ("codes", "block_scales", "col_scales", "tensor_scale", "mse"):
            assert torch.equal(r[k], g[k]), (fmt, k)


@pytest.mark.parametrize("fmt,group,col_dtype", PRIMARY)
def test_warm_start_rejects_inadmissible_scales(fmt, group, col_dtype):
    """An inadmissible given scale is found by the library's own check before any iteration runs:
    DQ_EINVAL from the device status, and the outputs past the given scales are untouched."""
    W = weight(32, 256, seed=11).cuda()
    base = _given(binding.dq_solve(W, fmt, group, 0, col_dtype))
    bad_a = {"int4": [0x0000, 0x7C00, 0x8001, 0x7E00], "mxint4": [0, 254, 255], "mxfp4": [0, 254, 255],
             "mxint8": [0, 254, 255], "mxfp8": [0, 254, 255],
             "nvfp4": [0x00, 0x7F, 0x80, 0xFF]}[fmt]
    cases = []
    for v in bad_a:
        s = {k: t.clone() for k, t in base.items()}
        blk = s["block_scales"]
        if fmt == "int4":
            blk.view(torch.int16).view(-1)[5] = v if v < 0x8000 else v - 0x10000
        else:
            blk.view(-1)[5] = v
        cases.append(s)
    for v in (0x0000, 0x7F80 if col_dtype == "bf16" else 0x7C00, 0x8001 - 0x10000):
        s = {k: t.clone() for k, t in base.items()}
        s["col_scales"].view(torch.int16)[7] = v
        cases.append(s)
    if fmt == "nvfp4":
        for v in (0.0, -1.0, float("inf"), float("nan")):
            s = {k: t.clone() for k, t in base.items()}
            s["tensor_scale"].fill_(v)
            cases.append(s)
    for s in cases:
        out = binding.alloc_outputs(32, 256, fmt, group, col_dtype, 2, "cuda")
        out["mse"].fill_(-1.0)
        with pytest.raises(binding.DQError) as e:
            binding.dq_solve(W, fmt, group, 2, col_dtype, init="given", init_scales=s, out=out)
        assert e.value.status == 1
        assert bool((out["mse"] == -1.0).all())


def test_workspace_bytes_ex():
    lib = binding.load_library()
    for rows, cols, fmt, g in ((14336, 4096, 2, 16), (4096, 14336, 1, 32), (16, 262144, 0, 64)):
        base = lib.dq_workspace_bytes(rows, cols, fmt, g)
        for init in (0, 2):
            assert lib.dq_workspace_bytes_ex(rows, cols, fmt, g, binding._Options(0, init, None)) == base
        l1 = lib.dq_workspace_bytes_ex(rows, cols, fmt, g, binding._Options(0, 1, None))
        assert l1 >= base and l1 >= 88 * cols
    W = weight(64, 512, seed=1).cuda()
    ws = torch.empty(lib.dq_workspace_bytes(64, 512, 2, 16), dtype=torch.uint8, device="cuda")
    need = lib.dq_workspace_bytes_ex(64, 512, 2, 16, binding._Options(0, 1, None))
    if need > ws.numel():
        with pytest.raises(binding.DQError) as e:
            binding.dq_solve(W, "nvfp4", 16, 1, "bf16", init="l1", workspace=ws)
        assert e.value.status == 3
