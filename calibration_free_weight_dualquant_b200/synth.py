"""Seeded synthetic weight matrices (Llama-shaped) for tests and benchmarks.

This module draws inputs only; it holds none of the solver's arithmetic, and
both the CUDA path and the CPU oracle are fed from it.  Recipe:

* values are drawn in fp32 from a numpy PCG64 generator seeded per workload,
  from N(0, sigma^2), a scaled Student-t, or a Laplace law;
* ``k = max(1, round_half_even(frac * N))`` distinct outlier columns, picked by
  a seeded permutation, are multiplied by a factor before the cast;
* the matrix is then rounded to bf16 (round to nearest even) unless the
  workload is fp32.

The pages measure on Llama-3.1-8B / Qwen checkpoints; with no checkpoint in
reach, these matrices of the same shapes stand in for them.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    rows: int
    cols: int
    wdtype: str          # "f32" | "bf16"
    fmt: str             # "int4" | "mxint4" | "nvfp4" | "mxfp4" | "mxint8"
    group: int
    col_dtype: str       # "f16" | "bf16"
    iters: int
    dist: str            # "normal" | "student_t" | "laplace"
    scale: float         # sigma, t multiplier, or Laplace scale
    outlier_frac: float
    outlier_mult: float
    seed: int
    df: float = 4.0
    note: str = ""


# The five workloads: one small fp32 matrix, three single Llama-shaped
# projections, and the full Llama-3.1-8B linear set (224 matrices).
WORKLOADS = {
    "int4_g64_256x512_f32": Workload(
        "int4_g64_256x512_f32", 256, 512, "f32", "int4", 64, "f16", 10, "normal", 0.02, 0.01, 20.0, 1001),
    "int4_g64_qproj_4096x4096": Workload(
        "int4_g64_qproj_4096x4096", 4096, 4096, "bf16", "int4", 64, "f16", 20, "normal", 0.02, 0.005, 15.0, 1002),
    "mxint4_g32_downproj_4096x14336": Workload(
        "mxint4_g32_downproj_4096x14336", 4096, 14336, "bf16", "mxint4", 32, "bf16", 20, "student_t", 0.015, 0.005,
        20.0, 1003),
    "nvfp4_g16_gateup_14336x4096": Workload(
        "nvfp4_g16_gateup_14336x4096", 14336, 4096, "bf16", "nvfp4", 16, "bf16", 30, "laplace", 0.012, 0.01, 10.0,
        1004),
    # the MX family's FP4 member on the down_proj recipe (a solver variant beyond the five configs)
    "mxfp4_g32_downproj_4096x14336": Workload(
        "mxfp4_g32_downproj_4096x14336", 4096, 14336, "bf16", "mxfp4", 32, "bf16", 20, "student_t", 0.015, 0.005,
        20.0, 1006),
    # the MX family's INT8 member (8-bit weights, DualQuant App. G.2) on the down_proj recipe
    "mxint8_g32_downproj_4096x14336": Workload(
        "mxint8_g32_downproj_4096x14336", 4096, 14336, "bf16", "mxint8", 32, "bf16", 20, "student_t", 0.015, 0.005,
        20.0, 1007),
    # the MX family's FP8 E4M3 member (8-bit weights, DualQuant App. G.2) on the down_proj recipe
    "mxfp8_g32_downproj_4096x14336": Workload(
        "mxfp8_g32_downproj_4096x14336", 4096, 14336, "bf16", "mxfp8", 32, "bf16", 20, "student_t", 0.015, 0.005,
        20.0, 1008),
}

# Llama-3.1-8B per-layer linear shapes (rows = out features, cols = in features)
LLAMA31_8B_LAYER = (("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096), ("o", 4096, 4096),
                    ("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336))
LLAMA31_8B_LAYERS = 32


def llama_set_workload(layer: int, proj_id: int, fmt: str, iters: int = 20) -> Workload:
    """One matrix of the 224-matrix Llama-3.1-8B linear set (N(0, 0.02^2), 0.5% outlier columns x15)."""
    name, rows, cols = LLAMA31_8B_LAYER[proj_id]
    group = 16 if fmt == "nvfp4" else 32
    seed = 5 * 10**6 + layer * 16 + proj_id
    return Workload("llama31_8b_L%d_%s_%s" % (layer, name, fmt), rows, cols, "bf16", fmt, group, "bf16", iters,
                    "normal", 0.02, 0.005, 15.0, seed)


def llama_set_elements() -> int:
    return LLAMA31_8B_LAYERS * sum(r * c for _, r, c in LLAMA31_8B_LAYER)


# The whole 224-matrix set, solved once per format (20 iterations each).
LLAMA_SETS = {"llama31_8b_set_nvfp4": "nvfp4", "llama31_8b_set_mxint4": "mxint4"}


def llama_set(fmt: str, iters: int = 20) -> list:
    """The 224 matrices in layer-major order (layer 0: q, k, v, o, gate, up, down; layer 1: ...)."""
    return [llama_set_workload(layer, pid, fmt, iters) for layer in range(LLAMA31_8B_LAYERS)
            for pid in range(len(LLAMA31_8B_LAYER))]


def make_weight_device(wl: Workload, device, seed: Optional[int] = None) -> torch.Tensor:
    """A normal-law workload drawn directly on `device` with torch's Philox generator seeded per matrix
    (the 14 GB Llama set is too large to draw on the host for every run).  Recipe: N(0, sigma^2) in fp32,
    k = max(1, round_half_even(frac N)) outlier columns chosen by a CPU torch permutation with the same
    seed and multiplied by the factor, then the round-to-nearest-even cast to bf16."""
    if wl.dist != "normal":
        raise ValueError("make_weight_device draws the normal law only")
    s = wl.seed if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(s)
    W = torch.randn((wl.rows, wl.cols), generator=gen, device=device, dtype=torch.float32) * wl.scale
    k = max(1, _round_half_even(wl.outlier_frac * wl.cols))
    cols = torch.randperm(wl.cols, generator=torch.Generator().manual_seed(s))[:k].to(device)
    W[:, cols] *= wl.outlier_mult
    return W.to(torch.bfloat16) if wl.wdtype == "bf16" else W


def _round_half_even(x: float) -> int:
    return int(np.round(x))  # numpy rounds half to even


def draw_fp32(wl: Workload, rows: Optional[int] = None, cols: Optional[int] = None, seed: Optional[int] = None
              ) -> np.ndarray:
    """The workload's fp32 draw (before the bf16 cast), optionally at another shape/seed."""
    M = wl.rows if rows is None else rows
    N = wl.cols if cols is None else cols
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    if wl.dist == "normal":
        W = rng.standard_normal((M, N), dtype=np.float32) * np.float32(wl.scale)
    elif wl.dist == "student_t":
        W = (rng.standard_t(wl.df, (M, N)) * wl.scale).astype(np.float32)
    elif wl.dist == "laplace":
        W = rng.laplace(0.0, wl.scale, (M, N)).astype(np.float32)
    else:
        raise ValueError(wl.dist)
    k = max(1, _round_half_even(wl.outlier_frac * N))
    cols_sel = rng.permutation(N)[:k]
    W[:, cols_sel] *= np.float32(wl.outlier_mult)
    return W


def make_weight(wl: Workload, rows: Optional[int] = None, cols: Optional[int] = None, seed: Optional[int] = None
                ) -> torch.Tensor:
    """CPU tensor [rows, cols] in the workload's dtype (bf16 via round-to-nearest-even cast)."""
    W = torch.from_numpy(draw_fp32(wl, rows, cols, seed))
    if wl.wdtype == "bf16":
        return W.to(torch.bfloat16)
    if wl.wdtype == "f16":
        return W.to(torch.float16)
    return W


def to_oracle_input(W: torch.Tensor):
    """(numpy array, wdtype) as the oracle takes it: f32 values, f16 values or bf16 bit patterns."""
    if W.dtype == torch.bfloat16:
        return W.contiguous().view(torch.int16).numpy().view(np.uint16), "bf16"
    if W.dtype == torch.float16:
        return W.contiguous().numpy(), "f16"
    return W.contiguous().numpy().astype(np.float32, copy=False), "f32"


def make_activations(tokens: int, cols: int, seed: int, outlier_frac: float = 0.01,
                     outlier_mult: float = 20.0) -> torch.Tensor:
    """Synthetic activations for the activation quantizer: N(0, 1) in fp32 (numpy PCG64), with
    k = max(1, round_half_even(frac * cols)) outlier channels (seeded permutation) multiplied by the
    factor -- the channel outliers that make activation quantization hard -- then cast to bf16 (RNE)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    X = rng.standard_normal((tokens, cols), dtype=np.float32)
    k = max(1, _round_half_even(outlier_frac * cols))
    X[:, rng.permutation(cols)[:k]] *= np.float32(outlier_mult)
    return torch.from_numpy(X).to(torch.bfloat16)


def make_col_scales(cols: int, seed: int) -> torch.Tensor:
    """Synthetic column inverse scales for the activation quantizer: exp(N(0, 0.3^2)) cast to bf16 (the
    solver's column scales stay within a small factor of 1)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return torch.from_numpy(np.exp(rng.normal(0.0, 0.3, cols)).astype(np.float32)).to(torch.bfloat16)
