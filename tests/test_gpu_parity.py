"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same seeded inputs.

Bar (spec tolerances): codes, block scales, column scales and the NVFP4
tensor scale bit-exact; every per-iteration MSE within 1e-4 relative.
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


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    binding.load_library()


def run_both(Wcpu: torch.Tensor, fmt, group, iters, col_dtype, label=""):
    gpu = binding.dq_solve(Wcpu.cuda(), fmt, group, iters, col_dtype)
    Win, wdt = synth.to_oracle_input(Wcpu)
    orc = oracle.solve(Win, wdt, fmt, group, iters, col_dtype)
    compare_with_oracle(fmt, gpu, orc, MSE_RTOL, label)
    return gpu, orc


# small shapes spanning several column strips, several CTAs per strip and a ragged tail
SMALL = {
    "int4_g64_256x512_f32": (333, 704),
    "int4_g64_qproj_4096x4096": (333, 704),
    "mxint4_g32_downproj_4096x14336": (301, 608),
    "nvfp4_g16_gateup_14336x4096": (339, 528),
    "mxfp4_g32_downproj_4096x14336": (301, 608),
    "mxint8_g32_downproj_4096x14336": (301, 608),
    "mxfp8_g32_downproj_4096x14336": (301, 608),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_parity_small_workload_recipe(name):
    wl = synth.WORKLOADS[name]
    M, N = SMALL[name]
    W = synth.make_weight(wl, M, N, seed=wl.seed + 7)
    gpu, orc = run_both(W, wl.fmt, wl.group, wl.iters, wl.col_dtype, name)
    mse = gpu["mse"].cpu().numpy()
    assert np.all(mse[1:] <= mse[:-1] * (1 + 1e-9))


@pytest.mark.parametrize("fmt,group,col_dtype,M,N,iters", [
    ("mxfp4", 32, "bf16", 999, 1088, 6),
    ("int4", 64, "f16", 1000, 1344, 6),
    ("mxint4", 32, "bf16", 777, 1056, 6),
    ("nvfp4", 16, "bf16", 1203, 800, 6),
    ("mxint8", 32, "bf16", 777, 1056, 6),
    ("mxfp8", 32, "bf16", 777, 1056, 6),
])
def test_parity_many_ctas(fmt, group, col_dtype, M, N, iters):
    wl = synth.WORKLOADS["nvfp4_g16_gateup_14336x4096"]
    W = synth.make_weight(wl, M, N, seed=77)
    run_both(W, fmt, group, iters, col_dtype, "many_ctas")


@pytest.mark.parametrize("fmt,group,col_dtype,M,N,wdtype", [
    ("mxfp4", 32, "bf16", 3, 32, torch.bfloat16),
    ("mxfp4", 32, "f16", 41, 288, torch.float32),
    ("int4", 8, "f16", 1, 8, torch.float32),
    ("int4", 256, "bf16", 5, 512, torch.bfloat16),
    ("int4", 128, "f16", 7, 384, torch.float16),
    ("mxint4", 32, "bf16", 2, 32, torch.float32),
    ("nvfp4", 16, "bf16", 3, 16, torch.bfloat16),
    ("nvfp4", 16, "f16", 65, 272, torch.float16),
    ("mxint8", 32, "bf16", 2, 32, torch.float32),
    ("mxint8", 32, "f16", 41, 288, torch.float16),
    ("mxint8", 32, "bf16", 3, 96, torch.bfloat16),
    ("mxfp8", 32, "bf16", 2, 32, torch.float32),
    ("mxfp8", 32, "f16", 41, 288, torch.float16),
    ("mxfp8", 32, "bf16", 3, 96, torch.bfloat16),
])
def test_parity_edge_shapes_and_dtypes(fmt, group, col_dtype, M, N, wdtype):
    g = torch.Generator().manual_seed(M * 1000 + N)
    W = (torch.randn(M, N, generator=g) * 0.05).to(wdtype)
    run_both(W, fmt, group, 5, col_dtype, "edge")


FORMATS = [("int4", 64, "f16"), ("mxint4", 32, "bf16"), ("nvfp4", 16, "bf16"), ("mxfp4", 32, "bf16"),
           ("mxint8", 32, "bf16"), ("mxfp8", 32, "bf16")]


@pytest.mark.parametrize("fmt,group,col_dtype", FORMATS)
def test_parity_zero_slices(fmt, group, col_dtype):
    g = torch.Generator().manual_seed(5)
    W = torch.randn(40, 4 * group, generator=g) * 0.02
    W[3, group:2 * group] = 0
    W[:, 5] = 0
    W[17] = 0
    run_both(W.to(torch.bfloat16), fmt, group, 6, col_dtype, "zero_slices")
    run_both(torch.zeros(9, 2 * group, dtype=torch.bfloat16), fmt, group, 3, col_dtype, "all_zero")


@pytest.mark.parametrize("fmt,group,col_dtype", FORMATS)
def test_parity_exact_ties(fmt, group, col_dtype):
    """Weights on a coarse dyadic lattice make exact rounding ties frequent."""
    g = torch.Generator().manual_seed(9)
    W = torch.randint(-24, 25, (64, 8 * group), generator=g).float() * 2.0 ** -7
    W[:, 3] *= 8
    run_both(W.to(torch.bfloat16), fmt, group, 8, col_dtype, "ties")


@pytest.mark.parametrize("fmt,group,col_dtype", FORMATS)
@pytest.mark.parametrize("mag", [1e-33, 1e-12, 1e4, 1e30])
def test_parity_extreme_magnitudes(fmt, group, col_dtype, mag):
    """Scales at the ends of the admissible sets (saturation, smallest values, fp64 fallback of the candidate)."""
    g = torch.Generator().manual_seed(11)
    W = torch.randn(16, 2 * group, generator=g) * mag
    W[:, 1] *= 1e3 if mag < 1 else 1.0
    run_both(W.float(), fmt, group, 4, col_dtype, "mag%g" % mag)


@pytest.mark.parametrize("fmt", ["int4", "mxint4", "nvfp4", "mxfp4", "mxint8", "mxfp8"])
def test_zero_iterations_is_rtn_and_deterministic(fmt):
    wl = synth.WORKLOADS["nvfp4_g16_gateup_14336x4096"]
    W = synth.make_weight(wl, 250, 1024, seed=3).cuda()
    r = binding.dq_rtn(W, fmt)
    s = binding.dq_solve(W, fmt, iters=0)
    for k in ("codes", "block_scales", "col_scales", "mse"):
        assert torch.equal(r[k], s[k]), k
    s1 = binding.dq_solve(W, fmt, iters=7)
    s2 = binding.dq_solve(W, fmt, iters=7)
    for k in ("codes", "block_scales", "col_scales", "mse", "tensor_scale"):
        assert torch.equal(s1[k], s2[k]), k
    assert float(s1["mse"][0]) == pytest.approx(float(r["mse"][0]), rel=1e-12)


def test_host_entry_point_matches_device():
    wl = synth.WORKLOADS["mxint4_g32_downproj_4096x14336"]
    W = synth.make_weight(wl, 96, 640, seed=4)
    host = binding.solve(W.pin_memory(), "mxint4", 32, 5, "bf16")
    dev = binding.dq_solve(W.cuda(), "mxint4", 32, 5, "bf16")
    for k in ("codes", "block_scales", "col_scales", "mse"):
        assert torch.equal(host[k], dev[k].cpu()), k


def test_nonfinite_input_reported():
    W = torch.zeros(8, 64, dtype=torch.bfloat16)
    W[2, 3] = float("nan")
    with pytest.raises(binding.DQError) as e:
        binding.dq_solve(W.cuda(), "int4", 64, 2, "f16")
    assert e.value.status == 4
    W[2, 3] = float("inf")
    with pytest.raises(binding.DQError) as e:
        binding.solve(W, "nvfp4", 16, 2)
    assert e.value.status == 4


def test_invalid_arguments_rejected_on_host():
    lib = binding.load_library()
    W = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    out = binding.alloc_outputs(4, 64, "int4", 64, "f16", 2, "cuda")
    o = binding._outputs_struct(out)
    ws = torch.empty(lib.dq_workspace_bytes(4, 64, 0, 64), dtype=torch.uint8, device="cuda")
    import ctypes
    s = torch.cuda.current_stream().cuda_stream

    def call(**kw):
        args = dict(W=W.data_ptr(), wdt=1, M=4, N=64, fmt=0, G=64, iters=2, cdt=2, ws=ws.data_ptr(),
                    wsb=ws.numel())
        args.update(kw)
        return lib.dq_solve(args["W"], args["wdt"], args["M"], args["N"], args["fmt"], args["G"], args["iters"],
                            args["cdt"], ctypes.byref(o), args["ws"], args["wsb"], s)

    assert call() == 0
    assert call(G=48) == 1            # cols not a multiple of group
    assert call(fmt=1, G=64) == 2     # MXINT4 needs group 32
    assert call(fmt=2, G=32) == 2     # NVFP4 needs group 16
    assert call(M=0) == 1
    assert call(N=63, G=7) == 1
    assert call(iters=-1) == 1
    assert call(wsb=ws.numel() - 1) == 3
    assert call(W=W.data_ptr() + 2) == 1   # W must be 16-byte aligned
    assert call(cdt=0) == 2
    assert call(G=24, N=72) == 2      # group must be a power of two in [8, 256]
    assert call(W=0) == 1
    assert lib.dq_workspace_bytes(4, 64, 1, 64) == 0
    torch.cuda.synchronize()


# ---------------------------------------------------------------------------
# Full sizes, in the launch configuration the benchmark times


def full_weight(name):
    wl = synth.WORKLOADS[name]
    return wl, synth.make_weight(wl)


def test_full_size_qproj_int4_against_full_oracle():
    """4096x4096 bf16 INT4-G64, 20 iterations: the whole solve against the oracle."""
    wl, W = full_weight("int4_g64_qproj_4096x4096")
    run_both(W, wl.fmt, wl.group, wl.iters, wl.col_dtype, wl.name)


@pytest.mark.parametrize("name", ["nvfp4_g16_gateup_14336x4096", "int4_g64_256x512_f32",
                                  "mxint4_g32_downproj_4096x14336", "mxfp4_g32_downproj_4096x14336",
                                  "mxint8_g32_downproj_4096x14336", "mxfp8_g32_downproj_4096x14336"])
def test_full_size_whole_trajectory(name):
    """Every full-size workload exactly as the benchmark runs it (its own shape, seed, law and
    iteration count; the 14336x4096 NVFP4 one is the headline workload): the whole solve against
    the oracle -- every per-iteration MSE within 1e-4, final codes, block scales, column scales and
    s_T bit-exact (reproduction README "Core equations"; the benchmark spec's tolerances) -- and the MSE
    never increases."""
    wl, W = full_weight(name)
    gpu, _ = run_both(W, wl.fmt, wl.group, wl.iters, wl.col_dtype, wl.name)
    mse = gpu["mse"].cpu().numpy()
    assert np.all(mse[1:] <= mse[:-1] * (1 + 1e-9))


@pytest.mark.parametrize("fmt,group,col_dtype,name", [
    ("int4", 64, "f16", "int4_g64_qproj_4096x4096"),
    ("mxint4", 32, "bf16", "mxint4_g32_downproj_4096x14336"),
    ("mxint8", 32, "bf16", "mxint8_g32_downproj_4096x14336"),
    ("mxfp8", 32, "bf16", "mxfp8_g32_downproj_4096x14336"),
])
def test_exact_paths_exercised_and_bit_exact(fmt, group, col_dtype, name):
    """The fp32 fast paths hand near-boundary elements, near-midpoint block scales and
    near-midpoint column scales to the exact paths; the result stays bit-exact."""
    wl = synth.WORKLOADS[name]
    W = synth.make_weight(wl, 1024, 2048, seed=5)
    gpu, _ = run_both(W, fmt, group, 20, col_dtype, "exact_paths")
    d = binding.diagnostics(gpu["workspace"])
    if fmt in ("mxint4", "mxint8", "mxfp8"):  # bf16 W, 2^k a: every flagged element is a certified exact tie
        assert d["quant_tie_lane_rows"] > 0, d
    else:
        assert d["quant_exact_lane_rows"] > 0, d
    if col_dtype == "f16":  # fp16 scales: near-midpoint LS values are common enough to be hit
        assert d["block_exact"] > 0 and d["col_exact"] > 0, d


def short_tensor_scale_weight(M, N, wdtype, seed):
    """Laplace weights whose max |W| is 2688 * 5 * 2^-13, so s_T = 5 * 2^-13 has 3 significant
    bits: a b then has few bits and many elements land exactly on E2M1 rounding boundaries."""
    rng = np.random.Generator(np.random.PCG64(seed))
    W = np.clip(rng.laplace(0.0, 0.012, (M, N)), -1.5, 1.5).astype(np.float32)
    W[M // 2, N // 3] = -2688.0 * 5.0 * 2.0 ** -13
    return torch.from_numpy(W).to(wdtype)


@pytest.mark.parametrize("wdtype,col_dtype,certified", [
    (torch.bfloat16, "bf16", True),    # 3 + 4 + 8 bits: certified ties
    (torch.float16, "bf16", True),
    (torch.float16, "f16", None),      # fp16 b: certified only on lanes whose b have few bits
    (torch.float32, "bf16", False),    # f32 W: never certified
])
def test_nvfp4_exact_ties(wdtype, col_dtype, certified):
    """Exact ties W / (a b) == boundary: certified lanes settle them on the fast path (round half
    to even in the code domain), the others on the exact path; both bit-exact."""
    W = short_tensor_scale_weight(517, 1040, wdtype, 11)
    gpu, orc = run_both(W, "nvfp4", 16, 6, col_dtype, "ties")
    assert orc["sT"] == 5.0 * 2.0 ** -13
    d = binding.diagnostics(gpu["workspace"])
    if certified:
        assert d["quant_tie_lane_rows"] > 0, d
    elif certified is None:
        assert d["quant_tie_lane_rows"] + d["quant_exact_lane_rows"] > 0, d
    else:
        assert d["quant_tie_lane_rows"] == 0 and d["quant_exact_lane_rows"] > 0, d


@pytest.mark.parametrize("wdtype,col_dtype", [(torch.float16, "f16"), (torch.bfloat16, "bf16"),
                                              (torch.float32, "bf16")])
def test_mxint4_exact_ties(wdtype, col_dtype):
    """MXINT4 with few-bit weights: W / (2^k b) hits half-integers exactly and often."""
    g = torch.Generator().manual_seed(12)
    W = (torch.randint(-40, 41, (389, 672), generator=g).float() * 2.0 ** -6).to(wdtype)
    gpu, _ = run_both(W, "mxint4", 32, 6, col_dtype, "mx_ties")
    d = binding.diagnostics(gpu["workspace"])
    if wdtype != torch.float32:
        assert d["quant_tie_lane_rows"] > 0, d
    else:
        assert d["quant_tie_lane_rows"] == 0, d


@pytest.mark.parametrize("mode", ["row", "col"])
@pytest.mark.parametrize("fmt,group,col_dtype", FORMATS)
def test_ablation_modes_parity(mode, fmt, group, col_dtype):
    """Row-only and column-only solves (DualQuant §5.3, Table 4) against the oracle's modes."""
    wl = synth.WORKLOADS["nvfp4_g16_gateup_14336x4096"]
    W = synth.make_weight(wl, 611, 1088, seed=91)
    gpu = binding.dq_solve(W.cuda(), fmt, group, 5, col_dtype, mode=mode)
    Win, wdt = synth.to_oracle_input(W)
    orc = oracle.solve(Win, wdt, fmt, group, 5, col_dtype, mode=mode)
    compare_with_oracle(fmt, gpu, orc, MSE_RTOL, mode)
    if mode == "row":
        assert bool((gpu["col_scales"].float() == 1).all())
    else:
        assert torch.equal(gpu["block_scales"], binding.dq_rtn(W.cuda(), fmt, group, col_dtype)["block_scales"])


def test_mxfp4_exact_ties():
    """MXFP4 on few-bit weights: W / (2^k b) hits E2M1 boundaries exactly; bf16 W and b make every
    flagged element a certified tie."""
    g = torch.Generator().manual_seed(14)
    W = (torch.randint(-48, 49, (389, 672), generator=g).float() * 2.0 ** -6).to(torch.bfloat16)
    gpu, _ = run_both(W, "mxfp4", 32, 6, "bf16", "mxfp4_ties")
    d = binding.diagnostics(gpu["workspace"])
    assert d["quant_tie_lane_rows"] > 0, d


@pytest.mark.parametrize("wdtype,col_dtype", [(torch.bfloat16, "bf16"), (torch.float16, "f16"),
                                              (torch.float32, "bf16")])
def test_mxint8_exact_ties(wdtype, col_dtype):
    """MXINT8 on half-integer lattices: every block holds the value 127 * 2^-8, so its RTN scale is
    exactly 2^-8 and every other W / a = m + 1/2 is an exact tie on the INT8 grid; certified on
    the fast path for bf16/fp16 W.  For f32 W nothing is certified: with a power-of-two b the
    candidate W * (1/b) * 2^-k is exact and its own round-half-even settles the tie."""
    g = torch.Generator().manual_seed(15)
    M, N = 203, 640
    m = torch.randint(-100, 100, (M, N), generator=g).float()
    W = (m + 0.5) * 2.0 ** -8
    W[:, ::32] = 127.0 * 2.0 ** -8
    gpu, _ = run_both(W.to(wdtype), "mxint8", 32, 6, col_dtype, "int8_ties")
    d = binding.diagnostics(gpu["workspace"])
    if wdtype != torch.float32:
        assert d["quant_tie_lane_rows"] > 0, d
    else:
        assert d["quant_tie_lane_rows"] == 0, d


def test_mxint8_grid_ends_and_clipping():
    """Values past both ends of the INT8 grid clip to -128 and 127 (two's-complement bytes 0x80, 0x7F)."""
    g = torch.Generator().manual_seed(16)
    W = torch.randn(64, 256, generator=g) * 0.01
    W[:, 0] = 0.5      # with the next column, the block scale: Proj(1/127) = 2^-7
    W[:, 1] = -1.0     # W/a = -128, the lower end
    W[:, 2] = 1.0      # W/a = 128 clips to 127
    gpu, orc = run_both(W.to(torch.bfloat16), "mxint8", 32, 0, "bf16", "int8_ends")
    codes = gpu["codes"].cpu()
    assert codes.shape == (64, 256)
    assert bool((codes[:, 1] == 0x80).all()) and bool((codes[:, 2] == 0x7F).all())


def e4m3_midpoints() -> torch.Tensor:
    """Midpoints of neighbouring nonnegative E4M3 values below 448 (from torch's float8_e4m3fn)."""
    v = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    return (v[:-1] + v[1:]) / 2


@pytest.mark.parametrize("wdtype,col_dtype", [(torch.bfloat16, "bf16"), (torch.float16, "f16"),
                                              (torch.float32, "bf16")])
def test_mxfp8_exact_ties(wdtype, col_dtype):
    """MXFP8 on E4M3 midpoints: every block holds 448 * 2^-8, so its RTN scale is exactly 2^-8 and
    every other W / a is a midpoint of two E4M3 values (an exact tie, subnormal ones included);
    certified on the fast path for bf16/fp16 W, settled exactly for f32 W."""
    g = torch.Generator().manual_seed(17)
    M, N = 203, 640
    mids = e4m3_midpoints()
    idx = torch.randint(0, len(mids), (M, N), generator=g)
    sign = torch.where(torch.rand(M, N, generator=g) < 0.5, -1.0, 1.0).double()
    W = (mids[idx] * sign * 2.0 ** -8).float()
    W[:, ::32] = 448.0 * 2.0 ** -8
    gpu, _ = run_both(W.to(wdtype), "mxfp8", 32, 6, col_dtype, "e4m3_ties")
    d = binding.diagnostics(gpu["workspace"])
    if wdtype != torch.float32:
        assert d["quant_tie_lane_rows"] > 0, d
    else:
        assert d["quant_tie_lane_rows"] == 0 and d["quant_exact_lane_rows"] > 0, d


def test_mxfp8_grid_ends_and_subnormals():
    """E4M3 saturation at +-448 (0x7E, 0xFE), the smallest subnormal 2^-9 (0x01), the midpoint 2^-10
    (a tie that goes to zero, code 0x00) and exact zeros (0x00, never 0x80)."""
    g = torch.Generator().manual_seed(18)
    W = torch.randn(64, 256, generator=g) * 0.01
    W[:, 0] = 1.75               # with the next column, the block scale: Proj(1.875 / 448) = 2^-8
    W[:, 1] = -1.75              # -448
    W[:, 2] = 1.875              # 480 clips to 448
    W[:, 3] = 2.0 ** -17         # 2^-9, the smallest subnormal
    W[:, 4] = -(2.0 ** -18)      # -2^-10: tie between 0 and -2^-9, to zero
    W[:, 5] = 0.0
    gpu, _ = run_both(W.to(torch.bfloat16), "mxfp8", 32, 0, "bf16", "e4m3_ends")
    codes = gpu["codes"].cpu()
    assert codes.shape == (64, 256)
    for col, want in ((1, 0xFE), (2, 0x7E), (3, 0x01), (4, 0x00), (5, 0x00)):
        assert bool((codes[:, col] == want).all()), (col, codes[:3, col].tolist())
