"""Brute-force and exact-rational references used to pin the oracle.

Nothing here reuses the oracle's arithmetic: admissible scale sets are
enumerated from library dtypes (numpy float16, bf16 bit patterns, torch
float8_e4m3fn), grid decisions are taken by exhaustive search with exact
rationals, and least-squares objectives are evaluated directly.
"""
from __future__ import annotations

from fractions import Fraction
from functools import lru_cache

import numpy as np
import torch

INT4_VALUES = list(range(-8, 8))
INT8_VALUES = list(range(-128, 128))
E2M1_MAGS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]  # encodings 0..7
E2M1_VALUES = sorted(set([-m for m in E2M1_MAGS] + E2M1_MAGS))


@lru_cache(maxsize=None)
def e4m3_values():
    """Every finite FP8 E4M3 value (torch float8_e4m3fn bit patterns 0x00..0x7E and their negatives,
    zero once), ascending, with the mantissa-bit-even flag of its encoding."""
    bits = np.arange(0, 0x7F, dtype=np.uint8)
    mags = torch.from_numpy(bits).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    even = {}
    for b, m in zip(bits.tolist(), mags.tolist()):
        even[m] = even[-m] = (b & 1) == 0
    vals = sorted(set(mags.tolist()) | set((-mags).tolist()))
    return vals, even


def grid_values(fmt: str):
    if fmt == "mxint8":
        return INT8_VALUES
    if fmt == "mxfp8":
        return e4m3_values()[0]
    return INT4_VALUES if fmt in ("int4", "mxint4") else E2M1_VALUES


def grid_qmax(fmt: str) -> int:
    """qmax of the absmax init: largest positive grid value."""
    return {"mxint8": 127, "nvfp4": 6, "mxfp4": 6, "mxfp8": 448}.get(fmt, 7)


def grid_is_even(fmt: str, v: float) -> bool:
    """Tie winner flag: even integer (INT4/INT8) or even mantissa bit of the E2M1 / E4M3 encoding."""
    if fmt in ("int4", "mxint4", "mxint8"):
        return int(v) % 2 == 0
    if fmt == "mxfp8":
        return e4m3_values()[1][float(v)]
    return E2M1_MAGS.index(abs(v)) % 2 == 0


def grid_argmin(fmt: str, w: float, ab: Fraction) -> float:
    """argmin over the grid of |w - ab*q| in exact rationals; ties to the even value."""
    W = Fraction(w)
    best, bestd = None, None
    for q in grid_values(fmt):
        d = abs(W - ab * Fraction(q))
        if best is None or d < bestd:
            best, bestd = q, d
        elif d == bestd:
            if grid_is_even(fmt, q):
                best = q
    return float(best)


@lru_cache(maxsize=None)
def enum_admissible(kind: str):
    """All admissible positive inverse scales of a format, ascending, with an 'even' flag per value."""
    if kind == "f16":
        bits = np.arange(1, 0x7C00, dtype=np.uint16)
        vals = bits.view(np.float16).astype(np.float64)
        even = (bits & 1) == 0
    elif kind == "bf16":
        bits = np.arange(1, 0x7F80, dtype=np.uint32)
        vals = (bits << 16).astype(np.uint32).view(np.float32).astype(np.float64)
        even = (bits & 1) == 0
    elif kind == "e4m3":
        bits = np.arange(1, 0x7F, dtype=np.uint8)  # 0x7F is NaN
        vals = torch.from_numpy(bits.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        even = (bits & 1) == 0
    elif kind == "e8m0":
        ks = np.arange(-126, 127)
        vals = np.ldexp(1.0, ks)
        even = np.zeros(len(ks), bool)  # ties go up, handled in nearest_admissible
    else:
        raise ValueError(kind)
    order = np.argsort(vals)
    return vals[order], even[order]


def nearest_admissible(kind: str, v: float) -> float:
    """Nearest admissible value to v in linear distance (exact compare); ties: even mantissa, or larger for e8m0."""
    vals, even = enum_admissible(kind)
    i = int(np.searchsorted(vals, v))
    cands = [k for k in (i - 1, i) if 0 <= k < len(vals)]
    V = Fraction(v)
    best = None
    for k in cands:
        d = abs(Fraction(float(vals[k])) - V)
        if best is None or d < best[0]:
            best = (d, k)
        elif d == best[0]:
            if kind == "e8m0":
                best = (d, max(best[1], k))
            elif even[k]:
                best = (d, k)
    return float(vals[best[1]])


def argmin_scale_objective(kind: str, W: np.ndarray, R: np.ndarray, scale_factor: float = 1.0) -> float:
    """argmin over admissible f of sum (W - scale_factor*f*R)^2, by exhaustive evaluation.

    Candidates within a hair of the fp64 minimum are re-ranked with exact
    rationals; an exact tie goes to the even mantissa (larger power for e8m0).
    Returns the admissible factor f.
    """
    vals, even = enum_admissible(kind)
    W = np.asarray(W, np.float64)
    R = np.asarray(R, np.float64)
    obj = np.zeros(len(vals))
    chunk = 4096
    for s in range(0, len(vals), chunk):
        f = vals[s:s + chunk, None] * scale_factor
        obj[s:s + chunk] = ((W[None, :] - f * R[None, :]) ** 2).sum(axis=1)
    m = obj.min()
    close = np.nonzero(obj <= m * (1 + 1e-9) + 1e-300)[0]
    Wf = [Fraction(float(x)) for x in W]
    Rf = [Fraction(float(x)) for x in R]
    sf = Fraction(scale_factor)
    best = None
    for k in close:
        f = Fraction(float(vals[k])) * sf
        o = sum((wv - f * rv) ** 2 for wv, rv in zip(Wf, Rf))
        if best is None or o < best[0]:
            best = (o, k)
        elif o == best[0]:
            if kind == "e8m0":
                best = (o, max(best[1], k))
            elif even[k]:
                best = (o, k)
    return float(vals[best[1]])


def decode_codes(fmt: str, codes: np.ndarray) -> np.ndarray:
    """Unpack nibble codes [M, N/2] -> grid values [M, N] (even column in the low nibble);
    MXINT8 codes [M, N] are one two's-complement byte each, MXFP8 codes [M, N] one E4M3 pattern each."""
    if fmt == "mxint8":
        return codes.view(np.int8).astype(np.float64)
    if fmt == "mxfp8":
        return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    lo = codes & 0xF
    hi = codes >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1).astype(np.int64)
    if fmt in ("int4", "mxint4"):
        return ((nib ^ 8) - 8).astype(np.float64)
    mag = np.array(E2M1_MAGS)[nib & 7]
    return np.where(nib & 8, -mag, mag)
