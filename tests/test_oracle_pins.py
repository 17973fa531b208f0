"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test cites the passage it checks.  None of them re-types the oracle's
formulas: they use printed values (tests/golden), exact rational arithmetic,
exhaustive enumeration of admissible scales, numpy least squares, and
invariants of the method.
"""
from __future__ import annotations

import os
import zlib
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import bruteforce as bf
from calibration_free_weight_dualquant_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

PROJ_KIND = {"f16": oracle.PROJ_F16, "bf16": oracle.PROJ_BF16, "e4m3": oracle.PROJ_E4M3, "e8m0": oracle.PROJ_E8M0}
A_KIND = {"int4": "f16", "mxint4": "e8m0", "nvfp4": "e4m3", "mxfp4": "e8m0", "mxint8": "e8m0", "mxfp8": "e8m0"}


def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            vals[k] = v
    return vals


def bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(
        np.uint16)


def bf16_values(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Printed examples


def test_int8_worked_example():
    """SQuant lesson, Ch. 2 'A fully worked int8 example': code 35, 0.13780, +0.00080, +0.20 ticks."""
    g = read_golden("int8_worked_example.txt")
    qmin, qmax = int(g["qmin"][0]), int(g["qmax"][0])
    grid = np.arange(qmin, qmax + 1, dtype=np.float64)
    even = (grid.astype(int) % 2 == 0).astype(np.uint8)
    s = oracle.absmax_scale([float(g["absmax"][0]), -0.3, 0.2], qmax)
    w = float(g["w"][0])
    code = int(grid[oracle.quant_index(w, s, grid, even)])
    assert code == int(g["code"][0])
    assert f"{w / s:.2f}" == g["w_over_s_2dp"][0]
    w_hat = code * s
    assert f"{w_hat:.5f}" == g["w_hat_5dp"][0]
    assert f"{w_hat - w:.5f}" == g["delta_w_5dp"][0]
    assert f"{code - w / s:.2f}" == g["ticks_2dp"][0]


def test_outlier_scale_example():
    """RTN tutorial, 'When RTN Fails': scale 100/127 ~ 0.79; [-1, 1] uses only levels -1, 0, +1."""
    g = read_golden("outlier_scale_example.txt")
    qmax = int(g["qmax"][0])
    rng = np.random.Generator(np.random.PCG64(7))
    x = np.concatenate([rng.uniform(-1, 1, 999), [float(g["outlier"][0])]])
    s = oracle.absmax_scale(x, qmax)
    assert f"{s:.2f}" == g["scale_2dp"][0]
    grid = np.arange(-qmax, qmax + 1, dtype=np.float64)
    even = (grid.astype(int) % 2 == 0).astype(np.uint8)
    levels = {int(grid[oracle.quant_index(v, s, grid, even)]) for v in x[:-1]}
    assert levels == {int(t) for t in g["levels_used"]}


def test_rtn_error_bound():
    """RTN tutorial, 'Round-to-Nearest (RTN)': |w - w_hat| <= s/2; tick error in [-0.5, 0.5] (SQuant Ch. 2)."""
    rng = np.random.Generator(np.random.PCG64(3))
    grid = np.arange(-8, 8, dtype=np.float64)
    even = (grid.astype(int) % 2 == 0).astype(np.uint8)
    for _ in range(20):
        w = rng.standard_normal(64) * 0.02
        s = oracle.absmax_scale(w, 7)
        q = np.array([grid[oracle.quant_index(v, s, grid, even)] for v in w])
        assert np.all(np.abs(w - q * s) <= s / 2 * (1 + 1e-15))
        ticks = q - w / s
        assert np.all(np.abs(ticks) <= 0.5 + 1e-12)


@pytest.mark.parametrize("fmt,qmax", [("mxint4", 7), ("mxfp4", 6), ("mxint8", 127), ("mxfp8", 448)])
def test_mx_rtn_scale_straddles_the_e8m0_midpoint(fmt, qmax):
    """Absmax RTN with power-of-two scales (RTN tutorial, 'Absmax (Symmetric) Quantization': scale
    max|w| / qmax, 127 for INT8; projected onto E8M0, ties up): a block whose absmax / qmax lies just
    above the midpoint 1.5 * 2^-8 gets 2^-7, just below it 2^-8.  The bands are 2^-10 relative wide,
    narrower than the step between neighbouring qmax values, so a wrong qmax moves one of them."""
    W = np.zeros((2, 64), np.float32)
    W[0, 5] = 1.5 * 2.0 ** -8 * qmax * (1 + 2.0 ** -10)
    W[1, 40] = -1.5 * 2.0 ** -8 * qmax * (1 - 2.0 ** -10)
    W[0, 33] = W[1, 7] = 1e-3  # the other block of each row: a small absmax
    out = oracle.rtn(W, "f32", fmt, 32, "bf16")
    assert out["a"][0, 0] == 2.0 ** -7 and out["a"][1, 1] == 2.0 ** -8, out["a"]


def test_storage_sizes():
    """DualQuant App. I / Table 12: 224 Llama-3.1-8B linears -> 3.49 GB codes + 0.22 GB G64 scales;
    RTN tutorial: g=128 fp16 scale overhead 3.1%."""
    g = read_golden("storage_sizes.txt")
    n = synth.llama_set_elements()
    assert synth.LLAMA31_8B_LAYERS * len(synth.LLAMA31_8B_LAYER) == 224
    # the oracle packs two codes per byte and emits one scale per 64-element group
    W = np.zeros((4, 128), np.float32)
    out = oracle.rtn(W, "f32", "int4", 64, "f16")
    assert out["codes"].size * 2 == W.size and out["a"].size * 64 == W.size
    codes_gb = n * out["codes"].size / W.size / 1e9
    scales_gb = n * out["a"].size * 2 / W.size / 1e9   # fp16 scales
    assert f"{codes_gb:.2f}" == g["llama31_8b_linear_packed_GB"][0]
    assert f"{scales_gb:.2f}" == g["llama31_8b_linear_g64_scales_GB"][0]
    out128 = oracle.rtn(np.zeros((4, 256), np.float32), "f32", "int4", 128, "f16")
    overhead = out128["a"].size * 2 / out128["codes"].size * 100
    assert f"{overhead:.1f}" == g["overhead_g128_fp16_percent_1dp"][0]


# ---------------------------------------------------------------------------
# Grid quantizer Q against exact rationals


@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "mxint8", "mxfp8"])
def test_quantizer_exact_rational(fmt):
    """Q = nearest grid value, ties to even, clip (DualQuant §3; reproduction README 'Local reproduction')."""
    rng = np.random.Generator(np.random.PCG64(11))
    vals, _ = bf.enum_admissible("f16")
    for trial in range(400):
        a = float(rng.choice(vals[(vals > 1e-3) & (vals < 10)]))
        b = float(np.float16(rng.uniform(0.25, 4)))
        ab = Fraction(a) * Fraction(b)
        if trial % 3 == 0:
            # exactly on a boundary: (grid midpoint) * a * b, when it is representable
            g = bf.grid_values(fmt)
            k = rng.integers(0, len(g) - 1)
            h = (Fraction(g[k]) + Fraction(g[k + 1])) / 2
            w = float(h * ab)
        else:
            span = {"mxint8": 200, "mxfp8": 600}.get(fmt, 10)  # past both ends of the grid
            x = rng.uniform(-span, span)
            if fmt == "mxfp8" and trial % 3 == 1:  # every binade, subnormals included
                x = float(np.sign(x)) * 2.0 ** rng.uniform(-12, 9.5)
            w = float(x * a * b)
        got = oracle.quant_value(fmt, w, float(ab))
        assert got == bf.grid_argmin(fmt, w, ab), (w, a, b)


def test_quantizer_tie_cases():
    """Round half to even on the INT4 grid and on the E2M1 mantissa; ends clip."""
    cases_int = {0.5: 0, 1.5: 2, 2.5: 2, -0.5: 0, -1.5: -2, 6.5: 6, 7.5: 7, 9.0: 7, -8.5: -8, -20: -8}
    for x, q in cases_int.items():
        assert oracle.quant_value("int4", x, 1.0) == q
    cases_fp4 = {0.25: 0, 0.75: 1, 1.25: 1, 1.75: 2, 2.5: 2, 3.5: 4, 5.0: 4, 7.0: 6, -5.0: -4, -0.25: 0}
    for x, q in cases_fp4.items():
        assert oracle.quant_value("nvfp4", x, 1.0) == q


def test_quantizer_e4m3_matches_library_cast():
    """The MXFP8 element grid is FP8 E4M3: inside its range, Q(x) with unit scale equals torch's
    round-to-nearest-even cast to float8_e4m3fn (binade interiors, midpoints, subnormals); beyond
    448 it clips.  Midpoint cases: 1.0625 lies between 1 (mantissa 0) and 1.125 (mantissa 1) -> 1;
    1.1875 -> 1.25; the subnormal midpoint 3 * 2^-10 -> 2^-8; 2^-10 -> 0."""
    rng = np.random.Generator(np.random.PCG64(21))
    xs = np.concatenate([np.sign(rng.uniform(-1, 1, 3000)) * 2.0 ** rng.uniform(-12, np.log2(448), 3000),
                         rng.uniform(-448, 448, 1000)]).astype(np.float32)
    vals, _ = bf.e4m3_values()
    v = np.array(vals)
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)   # exact in fp32
    xs = np.concatenate([xs, mids, -mids, np.float32([0.0, 448.0, -448.0])])
    want = torch.from_numpy(xs).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    for x, w in zip(xs.tolist(), want.tolist()):
        assert oracle.quant_value("mxfp8", x, 1.0) == w, (x, w)
    for x, q in {1.0625: 1.0, 1.1875: 1.25, 3 * 2.0 ** -10: 2.0 ** -8, 2.0 ** -10: 0.0, 464.0: 448.0,
                 1e6: 448.0, -1e6: -448.0, -2.0 ** -10: 0.0,
                 1.9375: 2.0,                   # across a binade end: 1.875 (mantissa 7) vs 2 (mantissa 0)
                 15 * 2.0 ** -10: 2.0 ** -6,    # largest subnormal 7 * 2^-9 vs smallest normal 2^-6
                 432.0: 448.0,                  # 416 (mantissa 5) vs 448 (mantissa 6)
                 -13 * 2.0 ** -10: -6 * 2.0 ** -9}.items():
        assert oracle.quant_value("mxfp8", x, 1.0) == q, x


# ---------------------------------------------------------------------------
# Projection onto admissible inverse scales vs exhaustive enumeration


@pytest.mark.parametrize("kind", ["f16", "bf16", "e4m3", "e8m0"])
def test_projection_exhaustive(kind):
    """Projection onto hardware-legal inverse scales (reproduction README 'Core equations';
    DualQuant App. B 'nearest representable value')."""
    vals, _ = bf.enum_admissible(kind)
    rng = np.random.Generator(np.random.PCG64(5))
    lo, hi = np.log2(vals[0]), np.log2(vals[-1])
    tests = list(2.0 ** rng.uniform(lo - 2, hi + 2, 3000))
    idx = rng.integers(0, len(vals) - 1, 500)
    tests += list((vals[idx] + vals[idx + 1]) / 2)            # exact midpoints
    tests += [vals[0] / 3, vals[0] / 2, vals[-1] * 1.01, vals[-1] * 1e6, 0.0]
    if kind == "e8m0":
        tests += [1.5 * 2.0 ** k for k in range(-20, 20)]
    for v in tests:
        got = oracle.project(PROJ_KIND[kind], float(v))
        want = bf.nearest_admissible(kind, float(v)) if v > 0 else vals[0]
        assert got == want, (kind, v, got, want)


@pytest.mark.parametrize("kind", ["f16", "bf16", "e4m3", "e8m0"])
def test_encode_matches_library(kind):
    vals, _ = bf.enum_admissible(kind)
    for v in vals[:: max(1, len(vals) // 500)]:
        bits = oracle.encode(PROJ_KIND[kind], float(v))
        if kind == "f16":
            assert bits == int(np.float16(v).view(np.uint16))
        elif kind == "bf16":
            assert bits == int(np.float32(v).view(np.uint32) >> 16)
        elif kind == "e4m3":
            assert bits == int(torch.tensor([v], dtype=torch.float64).to(torch.float8_e4m3fn).view(torch.uint8)[0])
        else:
            assert 2.0 ** (bits - 127) == v and 1 <= bits <= 253


# ---------------------------------------------------------------------------
# Whole iterations against brute force on tiny matrices

TINY = [
    ("int4", 64, "f16", 6, 128, "bf16", 4),
    ("int4", 16, "bf16", 5, 48, "f32", 3),
    ("mxint4", 32, "bf16", 6, 64, "bf16", 4),
    ("nvfp4", 16, "bf16", 6, 64, "bf16", 4),
    ("nvfp4", 16, "f16", 4, 32, "f32", 3),
    ("mxfp4", 32, "bf16", 6, 64, "bf16", 4),
    ("mxfp4", 32, "f16", 4, 64, "f32", 3),
    ("mxint8", 32, "bf16", 4, 64, "bf16", 3),
    ("mxfp8", 32, "bf16", 4, 64, "bf16", 3),
    ("mxfp8", 32, "f16", 4, 64, "f32", 3),
]


def stable_seed(*key) -> int:
    """A seed from a key that is the same in every process (str hashes are randomised)."""
    return zlib.crc32(repr(key).encode()) & 0xFFFF


def tiny_matrix(rows, cols, wdt, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    W = (rng.laplace(0, 0.02, (rows, cols))).astype(np.float32)
    W[:, rng.permutation(cols)[:2]] *= 12
    if wdt == "bf16":
        bits = bf16_bits(W)
        return bits, "bf16", bf16_values(bits).reshape(rows, cols)
    return W, "f32", W.astype(np.float64)


def brute_codes(fmt, Wv, a_val, b, G):
    M, N = Wv.shape
    q = np.zeros((M, N))
    for i in range(M):
        for j in range(N):
            ab = Fraction(float(a_val[i, j // G])) * Fraction(float(b[j]))
            q[i, j] = bf.grid_argmin(fmt, float(Wv[i, j]), ab)
    return q


@pytest.mark.parametrize("fmt,G,col_dt,M,N,wdt,iters", TINY)
def test_iterations_brute_force(fmt, G, col_dt, M, N, wdt, iters):
    """Every step of every iteration re-derived by brute force from the previous state
    (reproduction README flowchart and 'Core equations'; DualQuant §4.3, App. B)."""
    Win, wdtype, Wv = tiny_matrix(M, N, wdt, seed=stable_seed(fmt, G, M, N))
    out = oracle.solve(Win, wdtype, fmt, G, iters, col_dt, want_q=True, trace=True, changes=True)
    sT = out["sT"]
    akind = A_KIND[fmt]
    # init: absmax RTN with beta = 1; NVFP4 tensor scale fp32(amax / (6*448))
    qmax = float(bf.grid_qmax(fmt))
    if fmt == "nvfp4":
        assert sT == float(np.float32(np.abs(Wv).max() / 2688.0))
    assert np.all(out["trace_b"][0] == 1.0)
    for i in range(M):
        for g in range(N // G):
            m = np.abs(Wv[i, g * G:(g + 1) * G]).max()
            want = bf.nearest_admissible(akind, (m / qmax) / sT) if m > 0 else 1.0
            assert out["trace_a"][0][i, g] == want
    check_iterations(out, fmt, G, col_dt, Wv, iters)


def check_iterations(out, fmt, G, col_dt, Wv, iters):
    """Re-derive every step of every iteration by brute force from the traced state."""
    M, N = Wv.shape
    sT = out["sT"]
    akind = A_KIND[fmt]
    scale_factor = sT if fmt == "nvfp4" else 1.0
    q_prev = None
    for t in range(iters + 1):
        a_t = out["trace_a"][t]
        b_t = out["trace_b"][t]
        q_t = brute_codes(fmt, Wv, a_t * scale_factor, b_t, G)
        if "changes" in out:  # elements whose grid value changed in iteration t
            assert int(out["changes"][t]) == (0 if t == 0 else int(np.sum(q_t != q_prev))), t
        q_prev = q_t
        # MSE definition: mean (W - a q b)^2
        rec = np.repeat(a_t * scale_factor, G, axis=1) * q_t * b_t[None, :]
        np.testing.assert_allclose(out["mse"][t], np.mean((Wv - rec) ** 2), rtol=1e-12)
        if t == iters:
            np.testing.assert_array_equal(out["q"], q_t)
            np.testing.assert_array_equal(bf.decode_codes(fmt, out["codes"]), q_t)
            # a zero code is always the all-zero nibble (no E2M1 "-0")
            assert not np.any((out["codes"] & 0xF) == 8) or fmt not in ("nvfp4", "mxfp4")
            assert not np.any((out["codes"] >> 4) == 8) or fmt not in ("nvfp4", "mxfp4")
            break
        # row update with codes fixed: projected LS minimiser over the enumerated set
        a_next = out["trace_a"][t + 1]
        for i in range(M):
            for g in range(N // G):
                sl = slice(g * G, (g + 1) * G)
                R = q_t[i, sl] * b_t[sl]
                if np.all(R == 0):
                    want = 1.0
                else:
                    want = bf.argmin_scale_objective(akind, Wv[i, sl], R, scale_factor)
                assert a_next[i, g] == want, (t, i, g)
        # requantize with the new a and old b, then column update
        q_mid = brute_codes(fmt, Wv, a_next * scale_factor, b_t, G)
        b_next = out["trace_b"][t + 1]
        S = np.repeat(a_next * scale_factor, G, axis=1) * q_mid
        for j in range(N):
            if np.all(S[:, j] == 0):
                assert b_next[j] == 1.0
            else:
                assert b_next[j] == bf.argmin_scale_objective(col_dt, Wv[:, j], S[:, j]), (t, j)


@pytest.mark.parametrize("fmt,G,col_dt", [("int4", 64, "f16"), ("mxint4", 32, "bf16"), ("nvfp4", 16, "bf16"),
                                          ("mxint8", 32, "bf16"), ("mxfp8", 32, "bf16")])
def test_closed_form_is_least_squares(fmt, G, col_dt):
    """With codes fixed the unprojected update is the 1-D least-squares solution
    (reproduction README 'Core equations'; DualQuant App. B)."""
    Win, wdtype, Wv = tiny_matrix(8, 4 * G, "bf16", seed=21)
    st = oracle.rtn(Win, wdtype, fmt, G, col_dt)
    sT = st["sT"]
    q = oracle.requant(Win, wdtype, fmt, G, col_dt, sT, st["a"], st["b"])
    _, raw = oracle.row_update(Win, wdtype, fmt, G, col_dt, sT, q, st["b"])
    for i in range(Wv.shape[0]):
        for g in range(Wv.shape[1] // G):
            sl = slice(g * G, (g + 1) * G)
            R = (q[i, sl] * st["b"][sl])[:, None]
            if np.all(R == 0):
                assert np.isnan(raw[i, g])
                continue
            x, *_ = np.linalg.lstsq(R, Wv[i, sl], rcond=None)
            np.testing.assert_allclose(raw[i, g], x[0], rtol=1e-12)
    a_val = st["a"] * (sT if fmt == "nvfp4" else 1.0)
    _, rawb = oracle.col_update(Win, wdtype, fmt, G, col_dt, sT, q, st["a"])
    S = np.repeat(a_val, G, axis=1) * q
    for j in range(Wv.shape[1]):
        if np.all(S[:, j] == 0):
            assert np.isnan(rawb[j])
            continue
        x, *_ = np.linalg.lstsq(S[:, j:j + 1], Wv[:, j], rcond=None)
        np.testing.assert_allclose(rawb[j], x[0], rtol=1e-12)


# ---------------------------------------------------------------------------
# Invariants of the method


def small_workload(name, rows, cols, seed):
    wl = synth.WORKLOADS[name]
    W = synth.make_weight(wl, rows, cols, seed)
    return wl, synth.to_oracle_input(W)


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_zero_iterations_is_rtn_and_mse_monotone(name):
    """Zero BCD iterations equal absmax RTN; MSE never increases (each half-step is an exact
    block minimiser: DualQuant §4.3, App. C)."""
    wl, (Win, wdt) = small_workload(name, 48, 256, 99)
    r = oracle.rtn(Win, wdt, wl.fmt, wl.group, wl.col_dtype)
    s = oracle.solve(Win, wdt, wl.fmt, wl.group, 0, wl.col_dtype)
    for k in ("codes", "a", "b", "mse"):
        np.testing.assert_array_equal(r[k], s[k])
    s = oracle.solve(Win, wdt, wl.fmt, wl.group, 12, wl.col_dtype)
    np.testing.assert_array_equal(s["mse"][0], r["mse"][0])
    assert np.all(s["mse"][1:] <= s["mse"][:-1] * (1 + 1e-12))
    assert s["mse"][-1] < s["mse"][0]


@pytest.mark.parametrize("fmt,G,col_dt", [("int4", 64, "f16"), ("mxint4", 32, "bf16"), ("nvfp4", 16, "bf16"),
                                          ("mxint8", 32, "bf16"), ("mxfp8", 32, "bf16")])
def test_half_steps_monotone(fmt, G, col_dt):
    """Objective non-increasing after every half-step, not only after codes settle."""
    Win, wdtype, _ = tiny_matrix(32, 4 * G, "bf16", seed=31)
    st = oracle.rtn(Win, wdtype, fmt, G, col_dt)
    sT, a, b = st["sT"], st["a"], st["b"]
    q = oracle.requant(Win, wdtype, fmt, G, col_dt, sT, a, b)
    prev = oracle.mse(Win, wdtype, fmt, G, col_dt, sT, q, a, b)
    for _ in range(8):
        a, _ = oracle.row_update(Win, wdtype, fmt, G, col_dt, sT, q, b)
        for stage in range(2):
            cur = oracle.mse(Win, wdtype, fmt, G, col_dt, sT, q, a, b)
            assert cur <= prev * (1 + 1e-12)
            prev = cur
            q = oracle.requant(Win, wdtype, fmt, G, col_dt, sT, a, b)
            if stage == 0:
                cur = oracle.mse(Win, wdtype, fmt, G, col_dt, sT, q, a, b)
                assert cur <= prev * (1 + 1e-12)
                prev = cur
                b, _ = oracle.col_update(Win, wdtype, fmt, G, col_dt, sT, q, a)


@pytest.mark.parametrize("fmt,G,col_dt", [("int4", 16, "f16"), ("mxint4", 32, "bf16"), ("nvfp4", 16, "bf16")])
def test_fixed_point_is_stationary(fmt, G, col_dt):
    """At a fixed point every scale is the admissible minimiser given the rest
    (Theorem 1, DualQuant §4.3 / App. C), and one more iteration changes nothing."""
    Win, wdtype, Wv = tiny_matrix(6, 2 * G, "bf16", seed=41)
    out = oracle.solve(Win, wdtype, fmt, G, 80, col_dt, trace=True)
    ta, tb = out["trace_a"], out["trace_b"]
    fixed = [t for t in range(1, 81) if np.array_equal(ta[t], ta[t - 1]) and np.array_equal(tb[t], tb[t - 1])]
    assert fixed, "no fixed point within 80 iterations"
    t = fixed[0]
    a, b = ta[t], tb[t]
    a2, b2 = oracle.iterate(Win, wdtype, fmt, G, col_dt, out["sT"], a, b)
    np.testing.assert_array_equal(a2, a)
    np.testing.assert_array_equal(b2, b)
    sf = out["sT"] if fmt == "nvfp4" else 1.0
    q = brute_codes(fmt, Wv, a * sf, b, G)
    for i in range(Wv.shape[0]):
        for g in range(Wv.shape[1] // G):
            sl = slice(g * G, (g + 1) * G)
            R = q[i, sl] * b[sl]
            if np.any(R != 0):
                assert a[i, g] == bf.argmin_scale_objective(A_KIND[fmt], Wv[i, sl], R, sf)


@pytest.mark.parametrize("fmt,G,col_dt", [("int4", 64, "f16"), ("mxint4", 32, "bf16"), ("nvfp4", 16, "bf16"),
                                          ("mxint8", 32, "bf16"), ("mxfp8", 32, "bf16")])
def test_zero_slices(fmt, G, col_dt):
    """'Use scale 1 for an all-zero code slice' (reproduction README 'Core equations')."""
    Win, wdtype, Wv = tiny_matrix(8, 4 * G, "f32", seed=51)
    Win = Win.copy()
    Win[2, G:2 * G] = 0.0      # a zero block
    Win[:, 3] = 0.0            # a zero column
    out = oracle.solve(Win, "f32", fmt, G, 5, col_dt, want_q=True)
    assert out["a"][2, 1] == 1.0
    assert out["b"][3] == 1.0
    assert np.all(out["q"][2, G:2 * G] == 0) and np.all(out["q"][:, 3] == 0)
    z = oracle.solve(np.zeros((4, 2 * G), np.float32), "f32", fmt, G, 3, col_dt)
    assert z["sT"] == 1.0 and np.all(z["a"] == 1.0) and np.all(z["b"] == 1.0)
    assert np.all(z["codes"] == 0) and np.all(z["mse"] == 0.0)


@pytest.mark.parametrize("fmt,G,col_dt", [("int4", 64, "f16"), ("mxint4", 32, "bf16"), ("nvfp4", 16, "bf16"),
                                          ("mxint8", 32, "bf16"), ("mxfp8", 32, "bf16")])
def test_power_of_two_equivariance(fmt, G, col_dt):
    """W -> 2^k W scales the block inverse scales (or s_T) by 2^k and leaves codes and b unchanged."""
    Win, _, _ = tiny_matrix(16, 4 * G, "f32", seed=61)
    o1 = oracle.solve(Win, "f32", fmt, G, 6, col_dt)
    o2 = oracle.solve(Win * np.float32(4.0), "f32", fmt, G, 6, col_dt)
    np.testing.assert_array_equal(o1["codes"], o2["codes"])
    np.testing.assert_array_equal(o1["b"], o2["b"])
    if fmt == "nvfp4":
        assert o2["sT"] == 4 * o1["sT"]
        np.testing.assert_array_equal(o1["a"], o2["a"])
    else:
        np.testing.assert_array_equal(o1["a"] * 4, o2["a"])
    np.testing.assert_allclose(o2["mse"], 16 * o1["mse"], rtol=1e-12)


def test_sign_flip_nvfp4():
    """The E2M1 grid is symmetric: W -> -W flips the sign bit of every nonzero code."""
    Win, _, _ = tiny_matrix(16, 64, "f32", seed=71)
    o1 = oracle.solve(Win, "f32", "nvfp4", 16, 6, "bf16", want_q=True)
    o2 = oracle.solve(-Win, "f32", "nvfp4", 16, 6, "bf16", want_q=True)
    np.testing.assert_array_equal(o1["a"], o2["a"])
    np.testing.assert_array_equal(o1["b"], o2["b"])
    np.testing.assert_array_equal(o1["q"], -o2["q"])


@pytest.mark.parametrize("seed,wdt,mult", [(101, "f32", 1.0), (102, "bf16", 1.0), (103, "f32", 37.25),
                                           (104, "bf16", 3.0e-5)])
def test_nvfp4_tensor_scale_maps_amax_to_the_top_of_the_format(seed, wdt, mult):
    """NVFP4's one fp32 per-tensor scale (summary §3, the NVFP4 configuration: E2M1 elements with
    FP8-E4M3 block scales) is the factor that makes the largest magnitude of the two-level format,
    E2M1's 6 times E4M3's 448, reconstruct the tensor's max |W|.  Checked on the RTN iterate from its
    consequences, not from the formula: the block that holds max |W| gets e = 448 (the top of E4M3),
    that element's code is +-6 (the top of E2M1), its reconstruction a q b = s_T 448 6 equals max |W|
    to within the fp32 rounding of s_T, and no block scale leaves the E4M3 range.  A constant other
    than 6 * 448 (448 alone, 6 alone, 7 * 448) or a power-of-two rounding of s_T fails here."""
    Win, wdtype, Wv = tiny_matrix(24, 96, wdt, seed)
    if mult != 1.0:
        Wv = Wv * mult
        if wdt == "bf16":
            Win = bf16_bits(Wv.astype(np.float32))
            Wv = bf16_values(Win).reshape(Wv.shape)
        else:
            Win = Wv.astype(np.float32)
            Wv = Win.astype(np.float64)
    out = oracle.solve(Win, wdtype, "nvfp4", 16, 0, "bf16", want_q=True)
    sT, e, q = out["sT"], out["a"], out["q"]
    i, j = np.unravel_index(np.argmax(np.abs(Wv)), Wv.shape)
    amax = abs(float(Wv[i, j]))
    assert e[i, j // 16] == 448.0
    assert abs(q[i, j]) == 6.0 and np.sign(q[i, j]) == np.sign(Wv[i, j])
    assert abs(Fraction(sT) * 448 * 6 - Fraction(amax)) <= Fraction(amax) * Fraction(1, 2 ** 24)
    assert np.all(e <= 448.0) and np.all(e >= 2.0 ** -9)


@pytest.mark.parametrize("fmt,G,col_dt", [("int4", 64, "f16"), ("nvfp4", 16, "bf16")])
def test_permutation_equivariance(fmt, G, col_dt):
    """Permuting whole column groups (or rows) permutes every output the same way."""
    Win, _, _ = tiny_matrix(12, 4 * G, "f32", seed=81)
    o1 = oracle.solve(Win, "f32", fmt, G, 6, col_dt, want_q=True)
    perm_g = np.array([2, 0, 3, 1])
    cols = np.concatenate([np.arange(g * G, (g + 1) * G) for g in perm_g])
    o2 = oracle.solve(np.ascontiguousarray(Win[:, cols]), "f32", fmt, G, 6, col_dt, want_q=True)
    np.testing.assert_array_equal(o1["q"][:, cols], o2["q"])
    np.testing.assert_array_equal(o1["a"][:, perm_g], o2["a"])
    np.testing.assert_array_equal(o1["b"][cols], o2["b"])
    rows = np.random.Generator(np.random.PCG64(1)).permutation(12)
    o3 = oracle.solve(np.ascontiguousarray(Win[rows]), "f32", fmt, G, 6, col_dt, want_q=True)
    np.testing.assert_array_equal(o1["q"][rows], o3["q"])
    np.testing.assert_array_equal(o1["a"][rows], o3["a"])
    np.testing.assert_array_equal(o1["b"], o3["b"])


def test_mx_exponent_range():
    """MXINT4 block scales are powers of two with exponents in [-126, 126] (reproduction README)."""
    wl, (Win, wdt) = small_workload("mxint4_g32_downproj_4096x14336", 32, 256, 5)
    out = oracle.solve(Win, wdt, "mxint4", 32, 5, "bf16")
    k = np.log2(out["a"])
    assert np.all(k == np.round(k)) and np.all(k >= -126) and np.all(k <= 126)
    # absmax/7 below 2^-126 projects to the smallest admissible scale at init; the codes
    # are then all zero, so the first block update applies the zero-slice rule (scale 1)
    tiny = oracle.solve(np.full((2, 32), 1e-40, np.float32), "f32", "mxint4", 32, 2, "bf16", trace=True)
    assert np.all(tiny["trace_a"][0] == 2.0 ** -126)
    assert np.all(tiny["a"] == 1.0)


def test_nonfinite_rejected():
    W = np.zeros((2, 64), np.float32)
    W[1, 5] = np.inf
    with pytest.raises(oracle.OracleError):
        oracle.rtn(W, "f32", "int4", 64, "f16")


@pytest.mark.parametrize("fmt,G", [("int4", 64), ("mxint4", 32), ("nvfp4", 16), ("int4", 16), ("mxfp4", 32)])
def test_act_quant_brute_force(fmt, G):
    """Beta-folded activation quantization (DualQuant §4.4; README flowchart 'Scale X by column inverse
    scales, then quantize'): codes, group scales and tensor scale re-derived by brute force from
    X' = X diag(b) -- the product formed as an exact rational, scales by enumerating the admissible
    set, codes by enumerating the grid."""
    rows, cols = 3, 4 * G
    bits, xdt, Xv = tiny_matrix(rows, cols, "bf16", seed=G * 7 + len(fmt))
    rng = np.random.Generator(np.random.PCG64(G))
    b_bits = bf16_bits(np.exp(rng.normal(0.0, 0.5, cols)).astype(np.float32))
    b = bf16_values(b_bits)
    Xv = Xv.copy()
    Xv[1, :G] = 0.0  # an all-zero group gets scale 1
    bits = bf16_bits(Xv.astype(np.float32))
    out = oracle.act_quant(bits, "bf16", b, fmt, G)
    Xp = [[Fraction(float(Xv[i, j])) * Fraction(float(b[j])) for j in range(cols)] for i in range(rows)]
    qmax = Fraction(6 if fmt in ("nvfp4", "mxfp4") else 7)
    sT = 1.0
    if fmt == "nvfp4":
        amax = max(abs(v) for row in Xp for v in row)
        sT = float(np.float32(float(amax / 2688)))
        assert out["sT"] == sT
    for i in range(rows):
        for g in range(cols // G):
            m = max(abs(v) for v in Xp[i][g * G:(g + 1) * G])
            want = bf.nearest_admissible(A_KIND[fmt], float(m / qmax) / sT) if m > 0 else 1.0
            assert out["a"][i, g] == want, (i, g)
            av = Fraction(float(want)) * Fraction(sT)
            for j in range(g * G, (g + 1) * G):
                q = bf.grid_argmin(fmt, float(Xp[i][j]), av)
                assert bf.decode_codes(fmt, out["codes"])[i, j] == q, (i, j)


@pytest.mark.parametrize("mode", ["row", "col"])
@pytest.mark.parametrize("fmt,G,col_dt,M,N,wdt,iters", TINY[:4] + TINY[5:6])
def test_ablation_modes_brute_force(mode, fmt, G, col_dt, M, N, wdt, iters):
    """Ablation modes (DualQuant §5.3, Table 4): 'row' updates only the block scales (b stays 1),
    'col' only the column scales (a stays at its RTN value); each step re-derived by brute force, and
    the MSE never increases."""
    Win, wdtype, Wv = tiny_matrix(M, N, wdt, seed=stable_seed(mode, fmt, G, M, N))
    out = oracle.solve(Win, wdtype, fmt, G, iters, col_dt, want_q=True, trace=True, mode=mode)
    sf = out["sT"] if fmt == "nvfp4" else 1.0
    akind = A_KIND[fmt]
    for t in range(iters):
        a_t, b_t = out["trace_a"][t], out["trace_b"][t]
        q_t = brute_codes(fmt, Wv, a_t * sf, b_t, G)
        a_n, b_n = out["trace_a"][t + 1], out["trace_b"][t + 1]
        if mode == "row":
            assert np.all(b_n == 1.0)
            for i in range(M):
                for g in range(N // G):
                    sl = slice(g * G, (g + 1) * G)
                    R = q_t[i, sl] * b_t[sl]
                    want = 1.0 if np.all(R == 0) else bf.argmin_scale_objective(akind, Wv[i, sl], R, sf)
                    assert a_n[i, g] == want, (t, i, g)
        else:
            assert np.array_equal(a_n, out["trace_a"][0])
            S = np.repeat(a_t * sf, G, axis=1) * q_t
            for j in range(N):
                want = 1.0 if np.all(S[:, j] == 0) else bf.argmin_scale_objective(col_dt, Wv[:, j], S[:, j])
                assert b_n[j] == want, (t, j)
    q_T = brute_codes(fmt, Wv, out["trace_a"][iters] * sf, out["trace_b"][iters], G)
    np.testing.assert_array_equal(out["q"], q_T)
    assert np.all(out["mse"][1:] <= out["mse"][:-1] * (1 + 1e-12))


# ---------------------------------------------------------------------------
# Init variants: per-column L1-norm column scales (DualQuant §5.3) and warm start


def test_exact_abs_sum_is_fsum():
    """The exact magnitude sum, rounded once, equals math.fsum (Shewchuk's correctly rounded sum)."""
    import math
    rng = np.random.Generator(np.random.PCG64(7))
    # (2^64 - 1) * 2^-85 + (2^64 - 1) * 2^-149 in six fp32 values, then 2^-149: the last unit
    # carries through two full 64-bit words of 2^-149 units; the exact sum is 2^-21
    carry = np.array([(2 ** 24 - 1) * 2.0 ** -45, (2 ** 24 - 1) * 2.0 ** -69, (2 ** 16 - 1) * 2.0 ** -85,
                      (2 ** 24 - 1) * 2.0 ** -109, (2 ** 24 - 1) * 2.0 ** -133, (2 ** 16 - 1) * 2.0 ** -149,
                      2.0 ** -149], np.float32)
    cases = [
        rng.standard_normal(5000).astype(np.float32),
        (rng.standard_normal(3000) * np.exp2(rng.integers(-140, 120, 3000))).astype(np.float32),
        np.array([1.0, 2.0 ** -53], np.float32),                 # exact tie: stays at 1
        np.array([1.0, 2.0 ** -53, 2.0 ** -149], np.float32),    # just above the tie: rounds up
        np.array([1.0, 2.0 ** -52, 2.0 ** -53], np.float32),     # tie with an odd last bit: rounds up to even
        carry,
        np.array([2.0 ** 127, 2.0 ** 127, 2.0 ** -149], np.float32),
        np.full(70000, 2.0 ** -149, np.float32),                 # fp32 subnormals only
        np.zeros(9, np.float32),
    ]
    for x in cases:
        want = math.fsum(np.abs(x.astype(np.float64)))
        assert oracle.exact_abs_sum(x) == want, x[:4]
    assert oracle.exact_abs_sum(carry) == 2.0 ** -21
    bits = bf16_bits(rng.laplace(0, 0.01, 4096).astype(np.float32))
    v = bf16_values(bits)
    assert oracle.exact_abs_sum(v) == math.fsum(np.abs(v))


def l1_expected_init(Wv, fmt, G, col_dt):
    """The L1-norm init re-derived with independent primitives: math.fsum for the exact norms,
    enumeration of the admissible sets for every projection."""
    import math
    M, N = Wv.shape
    mu = math.fsum(np.abs(Wv).ravel()) / N
    b = np.ones(N)
    for j in range(N):
        c = math.fsum(np.abs(Wv[:, j]))
        if c != 0.0 and mu != 0.0:
            b[j] = bf.nearest_admissible(col_dt, c / mu)
    Q = np.abs(Wv) / b[None, :]
    amax = Q.max()
    sT = 1.0
    if fmt == "nvfp4" and amax > 0:
        sT = float(np.float32(amax / 2688.0))
    qmax = float(bf.grid_qmax(fmt))
    a = np.ones((M, N // G))
    for i in range(M):
        for g in range(N // G):
            m = Q[i, g * G:(g + 1) * G].max()
            if m > 0:
                a[i, g] = bf.nearest_admissible(A_KIND[fmt], (m / qmax) / sT) if fmt == "nvfp4" else \
                    bf.nearest_admissible(A_KIND[fmt], m / qmax)
    return a, b, sT


@pytest.mark.parametrize("fmt,G,col_dt,M,N,wdt,iters", TINY[:4] + TINY[5:6])
def test_l1_init_brute_force(fmt, G, col_dt, M, N, wdt, iters):
    """L1-norm init re-derived independently, then every iteration by brute force; MSE non-increasing."""
    Win, wdtype, Wv = tiny_matrix(M, N, wdt, seed=stable_seed("l1", fmt, G, M, N))
    out = oracle.solve(Win, wdtype, fmt, G, iters, col_dt, want_q=True, trace=True, init="l1", changes=True)
    a0, b0, sT = l1_expected_init(Wv, fmt, G, col_dt)
    assert out["sT"] == sT
    np.testing.assert_array_equal(out["trace_b"][0], b0)
    np.testing.assert_array_equal(out["trace_a"][0], a0)
    assert not np.all(b0 == 1.0)  # the outlier columns get larger column scales
    check_iterations(out, fmt, G, col_dt, Wv, iters)
    assert np.all(out["mse"][1:] <= out["mse"][:-1] * (1 + 1e-12))


def equal_norm_matrix(M, N, seed):
    """Every column a signed permutation of one vector: all column L1 norms are equal."""
    rng = np.random.Generator(np.random.PCG64(seed))
    v = rng.laplace(0, 0.02, M).astype(np.float32)
    cols = [rng.permutation(v) * rng.choice(np.array([-1, 1], np.float32), M) for _ in range(N)]
    return np.ascontiguousarray(np.stack(cols, axis=1))


@pytest.mark.parametrize("fmt,G,col_dt", [("int4", 64, "f16"), ("mxint4", 32, "bf16"), ("nvfp4", 16, "bf16"),
                                          ("mxfp4", 32, "bf16")])
def test_l1_init_with_equal_column_norms_is_rtn(fmt, G, col_dt):
    """Equal column L1 norms give b = 1, and then the L1 init is the absmax RTN init bit for bit."""
    W = equal_norm_matrix(24, 4 * G, seed=11)
    r = oracle.solve(W, "f32", fmt, G, 5, col_dt)
    s = oracle.solve(W, "f32", fmt, G, 5, col_dt, init="l1")
    for k in ("codes", "a", "b", "mse"):
        np.testing.assert_array_equal(r[k], s[k])
    assert r["sT"] == s["sT"]


@pytest.mark.parametrize("fmt,G,col_dt", [("int4", 64, "f16"), ("mxint4", 32, "bf16"), ("nvfp4", 16, "bf16"),
                                          ("mxfp4", 32, "bf16")])
def test_l1_init_power_of_two_columns(fmt, G, col_dt):
    """Columns of an equal-norm matrix B scaled by s_j in {1, 1, 2, 4} (mean 2): the L1 init gives
    b = s/2 exactly and sees W D_b^-1 = 2B, so its block scales, tensor scale and codes are those of
    the absmax RTN init of 2B."""
    B = equal_norm_matrix(16, 4 * G, seed=12)
    s = np.tile(np.array([1, 1, 2, 4], np.float32), G)
    o = oracle.solve(B * s[None, :], "f32", fmt, G, 0, col_dt, init="l1")
    r = oracle.solve(B * np.float32(2), "f32", fmt, G, 0, col_dt)
    np.testing.assert_array_equal(o["b"], s / 2)
    np.testing.assert_array_equal(o["a"], r["a"])
    np.testing.assert_array_equal(o["codes"], r["codes"])
    assert o["sT"] == r["sT"]


@pytest.mark.parametrize("fmt,G,col_dt", [("int4", 64, "f16"), ("nvfp4", 16, "bf16")])
def test_l1_init_zero_columns_and_power_of_two_scaling(fmt, G, col_dt):
    """An all-zero column keeps b = 1 (zero-slice rule); an all-zero W gives scale 1 everywhere;
    W -> 4W leaves b and the codes unchanged under the L1 init."""
    Win, _, _ = tiny_matrix(12, 4 * G, "f32", seed=13)
    Win = Win.copy()
    Win[:, 5] = 0.0
    o = oracle.solve(Win, "f32", fmt, G, 4, col_dt, init="l1", want_q=True)
    assert o["b"][5] == 1.0 and np.all(o["q"][:, 5] == 0)
    z = oracle.solve(np.zeros((4, 2 * G), np.float32), "f32", fmt, G, 2, col_dt, init="l1")
    assert z["sT"] == 1.0 and np.all(z["a"] == 1.0) and np.all(z["b"] == 1.0) and np.all(z["mse"] == 0)
    o4 = oracle.solve(Win * np.float32(4), "f32", fmt, G, 4, col_dt, init="l1", want_q=True)
    np.testing.assert_array_equal(o["b"], o4["b"])
    np.testing.assert_array_equal(o["q"], o4["q"])


@pytest.mark.parametrize("init", ["rtn", "l1"])
@pytest.mark.parametrize("fmt,G,col_dt", [("int4", 64, "f16"), ("mxint4", 32, "bf16"), ("nvfp4", 16, "bf16"),
                                          ("mxfp4", 32, "bf16")])
def test_warm_start_continues_the_iteration(init, fmt, G, col_dt):
    """The iterate is the pair of scales (codes are a function of them), so T1 iterations followed by a
    warm start of T2 more equal T1 + T2 iterations: every output, and the MSE sequence from T1 on."""
    wl, (Win, wdt) = small_workload("nvfp4_g16_gateup_14336x4096", 40, 4 * 64, 17)
    full = oracle.solve(Win, wdt, fmt, G, 7, col_dt, init=init, changes=True)
    first = oracle.solve(Win, wdt, fmt, G, 3, col_dt, init=init)
    warm = oracle.solve(Win, wdt, fmt, G, 4, col_dt, init="given", a0=first["a"], b0=first["b"],
                        sT0=first["sT"], changes=True)
    for k in ("codes", "a", "b"):
        np.testing.assert_array_equal(full[k], warm[k])
    assert full["sT"] == warm["sT"]
    np.testing.assert_array_equal(full["mse"][3:], warm["mse"])
    np.testing.assert_array_equal(full["changes"][4:], warm["changes"][1:])


@pytest.mark.parametrize("fmt,G,col_dt", [("int4", 64, "f16"), ("mxint4", 32, "bf16"), ("nvfp4", 16, "bf16"),
                                          ("mxint8", 32, "bf16"), ("mxfp8", 32, "bf16")])
def test_warm_start_rejects_inadmissible_scales(fmt, G, col_dt):
    """A warm start takes only admissible scales: elements of F_a and F_b, a positive fp32 s_T."""
    wl, (Win, wdt) = small_workload("nvfp4_g16_gateup_14336x4096", 8, 2 * 64, 19)
    r = oracle.rtn(Win, wdt, fmt, G, col_dt)
    ok = dict(a0=r["a"], b0=r["b"], sT0=r["sT"])
    oracle.solve(Win, wdt, fmt, G, 1, col_dt, init="given", **ok)
    bad_a = {"int4": 1.0 + 2.0 ** -12, "mxint4": 0.75, "nvfp4": 1.0625, "mxint8": 0.75, "mxfp8": 0.75}[fmt]
    cases = [dict(ok, a0=np.where(np.arange(r["a"].size).reshape(r["a"].shape) == 3, bad_a, r["a"])),
             dict(ok, a0=-r["a"]), dict(ok, a0=r["a"] * 0.0),
             dict(ok, b0=np.where(np.arange(r["b"].size) == 2, 1.0 + 2.0 ** -14, r["b"])),
             dict(ok, b0=np.full_like(r["b"], np.nan))]
    if fmt == "nvfp4":
        cases += [dict(ok, sT0=0.0), dict(ok, sT0=0.1), dict(ok, sT0=float("inf"))]
    for c in cases:
        with pytest.raises(oracle.OracleError):
            oracle.solve(Win, wdt, fmt, G, 1, col_dt, init="given", **c)


def test_changes_vanish_at_a_fixed_point():
    """Once the iterate stops moving no code changes: the count is 0 from then on."""
    wl, (Win, wdt) = small_workload("mxint4_g32_downproj_4096x14336", 16, 128, 23)
    o = oracle.solve(Win, wdt, "mxint4", 32, 60, "bf16", trace=True, changes=True)
    still = [t for t in range(1, 61) if np.array_equal(o["trace_a"][t], o["trace_a"][t - 1])
             and np.array_equal(o["trace_b"][t], o["trace_b"][t - 1])]
    assert still, "no fixed point reached"
    for t in still:
        assert o["changes"][t] == 0
    assert o["changes"][0] == 0 and o["changes"][1] > 0
