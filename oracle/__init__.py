"""Plain fp64 CPU oracle of the DualQuant dual-scale BCD solver.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product path (the CUDA
library and its Python binding) never imports this package, and this package
imports nothing from the product.

The arithmetic lives in ``dq_oracle.c`` (plain loops, fp64); this module only
builds it with gcc and marshals numpy arrays through ctypes.  See the header of
``dq_oracle.c`` for the pages each step follows and the readings taken where
they are silent.

Functions with no external pin: the final reconstruction MSE values on the
synthetic workloads (no page prints one) -- parity unpinned for those values;
every step that produces them is pinned on small inputs by the tests.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libdq_oracle.so")

# numbering of formats, dtypes and projection kinds used by dq_oracle.c
INT4, MXINT4, NVFP4, MXFP4 = 0, 1, 2, 3
F32, BF16, F16 = 0, 1, 2
PROJ_F16, PROJ_BF16, PROJ_E4M3, PROJ_E8M0 = 0, 1, 2, 3
MXINT8, MXFP8 = 4, 5
FORMATS = {"int4": INT4, "mxint4": MXINT4, "nvfp4": NVFP4, "mxfp4": MXFP4, "mxint8": MXINT8, "mxfp8": MXFP8}
BYTE_CODE_FORMATS = ("mxint8", "mxfp8")  # one byte per code; the others pack two nibbles per byte
WDTYPES = {"f32": F32, "bf16": BF16, "f16": F16}

_lib = None


def build(force: bool = False) -> str:
    """Compile dq_oracle.c into libdq_oracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        D = ctypes.c_double
        lib.dqo_solve.argtypes = [P, I, I64, I64, I, I, I, I, P, P, P, P, P, P, P, P]
        lib.dqo_solve.restype = I
        lib.dqo_solve_mode.argtypes = [P, I, I64, I64, I, I, I, I, I, P, P, P, P, P, P, P, P]
        lib.dqo_solve_mode.restype = I
        lib.dqo_solve_ex.argtypes = [P, I, I64, I64, I, I, I, I, I, I, P, P, D, P, P, P, P, P, P, P, P, P]
        lib.dqo_solve_ex.restype = I
        lib.dqo_exact_abs_sum.argtypes = [P, I64]
        lib.dqo_exact_abs_sum.restype = D
        lib.dqo_step.argtypes = [P, I, I64, I64, I, I, I, D, I, P, P, P, P, P, P]
        lib.dqo_step.restype = I
        lib.dqo_project.argtypes = [I, D]
        lib.dqo_project.restype = D
        lib.dqo_encode.argtypes = [I, D]
        lib.dqo_encode.restype = ctypes.c_uint32
        lib.dqo_quant_index.argtypes = [D, D, P, P, I]
        lib.dqo_quant_index.restype = I
        lib.dqo_quant_value.argtypes = [I, D, D]
        lib.dqo_quant_value.restype = D
        lib.dqo_absmax_scale.argtypes = [P, I64, D]
        lib.dqo_absmax_scale.restype = D
        lib.dqo_num_threads.argtypes = []
        lib.dqo_num_threads.restype = I
        lib.dqo_set_num_threads.argtypes = [I]
        lib.dqo_set_num_threads.restype = None
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _as_input(W: np.ndarray, wdtype: str) -> np.ndarray:
    if wdtype == "f32":
        return np.ascontiguousarray(W, dtype=np.float32)
    if wdtype == "f16":
        return np.ascontiguousarray(W.view(np.uint16) if W.dtype == np.float16 else W, dtype=np.uint16)
    if wdtype == "bf16":
        if W.dtype != np.uint16:
            raise TypeError("bf16 input must be given as uint16 bit patterns")
        return np.ascontiguousarray(W)
    raise ValueError(wdtype)


def _check(st: int):
    if st != 0:
        raise OracleError("oracle status %d" % st)


MODES = {"dual": 0, "row": 1, "col": 2}
INITS = {"rtn": 0, "l1": 1, "given": 2}


def solve(W: np.ndarray, wdtype: str, fmt: str, group: int, iters: int, col_dtype: str,
          want_q: bool = False, trace: bool = False, mode: str = "dual", init: str = "rtn",
          a0: Optional[np.ndarray] = None, b0: Optional[np.ndarray] = None, sT0: float = 1.0,
          changes: bool = False) -> dict:
    """Run the full solver.  W is [M, N] (float32, float16, or uint16 bf16 bits).
    ``mode``: "dual" (the BCD iteration), or the ablation modes of DualQuant §5.3 / Table 4:
    "row" (block scales only, b keeps its initial value) and "col" (column scales only, a keeps
    its initial value).
    ``init``: "rtn" (absmax RTN, b = 1), "l1" (per-column L1-norm column scales, DualQuant §5.3),
    or "given" (warm start from stored block scales a0 [M, N/G], column scales b0 [N] and, for
    NVFP4, the tensor scale sT0).

    Returns codes [M, N/2] uint8 ([M, N] for MXINT8 and MXFP8), a [M, N/G] (stored block-scale values: fp16
    value, 2^k, or E4M3 value e for NVFP4), b [N], sT (NVFP4 tensor scale, 1
    otherwise), mse [iters+1]; optionally q [M, N] grid values, per-iteration
    traces of a and b, and changes [iters+1] (elements whose grid value changed
    in each iteration).
    """
    lib = _load()
    Win = _as_input(W, wdtype)
    M, N = Win.shape
    nb = N // group
    codes = np.zeros((M, N if fmt in BYTE_CODE_FORMATS else N // 2), np.uint8)
    a = np.zeros((M, nb), np.float64)
    b = np.zeros(N, np.float64)
    sT = np.zeros(1, np.float64)
    mse = np.zeros(iters + 1, np.float64)
    q = np.zeros((M, N), np.float64) if want_q else None
    ta = np.zeros((iters + 1, M, nb), np.float64) if trace else None
    tb = np.zeros((iters + 1, N), np.float64) if trace else None
    ch = np.zeros(iters + 1, np.uint64) if changes else None
    a0c = None if a0 is None else np.ascontiguousarray(a0, np.float64).reshape(M, nb)
    b0c = None if b0 is None else np.ascontiguousarray(b0, np.float64).reshape(N)
    st = lib.dqo_solve_ex(_ptr(Win), WDTYPES[wdtype], M, N, FORMATS[fmt], group, iters,
                          WDTYPES[col_dtype], MODES[mode], INITS[init], _ptr(a0c), _ptr(b0c), float(sT0),
                          _ptr(codes), _ptr(a), _ptr(b), _ptr(sT), _ptr(mse), _ptr(q), _ptr(ta), _ptr(tb), _ptr(ch))
    _check(st)
    out = {"codes": codes, "a": a, "b": b, "sT": float(sT[0]), "mse": mse}
    if want_q:
        out["q"] = q
    if trace:
        out["trace_a"] = ta
        out["trace_b"] = tb
    if changes:
        out["changes"] = ch
    return out


def exact_abs_sum(x: np.ndarray) -> float:
    """sum |x_k| of fp32-representable values, exact and rounded once to fp64."""
    xd = np.ascontiguousarray(x, np.float64).reshape(-1)
    return float(_load().dqo_exact_abs_sum(_ptr(xd), xd.size))


def rtn(W: np.ndarray, wdtype: str, fmt: str, group: int, col_dtype: str, want_q: bool = False) -> dict:
    """Absmax round-to-nearest with beta = 1 (the solver's initial iterate)."""
    return solve(W, wdtype, fmt, group, 0, col_dtype, want_q=want_q)


def values(W: np.ndarray, wdtype: str) -> np.ndarray:
    """Exact fp64 values of an input array given as the oracle takes it."""
    if wdtype == "bf16":
        return (np.ascontiguousarray(W, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if wdtype == "f16":
        return (W.view(np.float16) if W.dtype == np.uint16 else W.astype(np.float16)).astype(np.float64)
    return np.asarray(W, dtype=np.float32).astype(np.float64)


def act_quant(X: np.ndarray, xdtype: str, b: np.ndarray, fmt: str, group: int) -> dict:
    """Beta-folded activation quantization (DualQuant summary §4.4 'Inference-time procedure and
    overhead'; reproduction README flowchart, 'Scale X by column inverse scales, then quantize'):
    X' = X diag(b), formed exactly in fp64, then the format's row-wise absmax round-to-nearest of X'
    (`rtn`: group scale Proj(absmax/qmax), 1 for an all-zero group, NVFP4 tensor scale
    fp32(amax/2688)).  With bf16/fp16 X and b every x*b has at most 22 significant bits, so the f32
    copy handed to `rtn` is exact (checked)."""
    Xp = values(X, xdtype) * np.asarray(b, dtype=np.float64)[None, :]
    Xp32 = Xp.astype(np.float32)
    if not np.array_equal(Xp32.astype(np.float64), Xp):
        raise OracleError("x * b is not exact in fp32")
    return rtn(Xp32, "f32", fmt, group, "bf16")


def requant(W, wdtype, fmt, group, col_dtype, sT, a, b) -> np.ndarray:
    """Q(W/(a b)) for every element -> grid values [M, N]."""
    lib = _load()
    Win = _as_input(W, wdtype)
    M, N = Win.shape
    a = np.ascontiguousarray(a, np.float64).copy()
    b = np.ascontiguousarray(b, np.float64).copy()
    q = np.zeros((M, N), np.float64)
    _check(lib.dqo_step(_ptr(Win), WDTYPES[wdtype], M, N, FORMATS[fmt], group, WDTYPES[col_dtype], sT, 0,
                        _ptr(a), _ptr(b), None, _ptr(q), None, None))
    return q


def row_update(W, wdtype, fmt, group, col_dtype, sT, q, b):
    """Closed-form block update with codes fixed -> (stored a, unprojected LS values)."""
    lib = _load()
    Win = _as_input(W, wdtype)
    M, N = Win.shape
    a = np.zeros((M, N // group), np.float64)
    raw = np.zeros((M, N // group), np.float64)
    q = np.ascontiguousarray(q, np.float64)
    b = np.ascontiguousarray(b, np.float64).copy()
    _check(lib.dqo_step(_ptr(Win), WDTYPES[wdtype], M, N, FORMATS[fmt], group, WDTYPES[col_dtype], sT, 1,
                        _ptr(a), _ptr(b), _ptr(q), None, _ptr(raw), None))
    return a, raw


def col_update(W, wdtype, fmt, group, col_dtype, sT, q, a):
    """Closed-form column update with codes fixed -> (b, unprojected LS values)."""
    lib = _load()
    Win = _as_input(W, wdtype)
    M, N = Win.shape
    b = np.zeros(N, np.float64)
    raw = np.zeros(N, np.float64)
    q = np.ascontiguousarray(q, np.float64)
    a = np.ascontiguousarray(a, np.float64).copy()
    _check(lib.dqo_step(_ptr(Win), WDTYPES[wdtype], M, N, FORMATS[fmt], group, WDTYPES[col_dtype], sT, 2,
                        _ptr(a), _ptr(b), _ptr(q), None, _ptr(raw), None))
    return b, raw


def iterate(W, wdtype, fmt, group, col_dtype, sT, a, b, want_q: bool = False):
    """One full BCD iteration from the state (a, b) -> (a', b'[, q'])."""
    lib = _load()
    Win = _as_input(W, wdtype)
    M, N = Win.shape
    a = np.ascontiguousarray(a, np.float64).copy()
    b = np.ascontiguousarray(b, np.float64).copy()
    q = np.zeros((M, N), np.float64) if want_q else None
    _check(lib.dqo_step(_ptr(Win), WDTYPES[wdtype], M, N, FORMATS[fmt], group, WDTYPES[col_dtype], sT, 3,
                        _ptr(a), _ptr(b), None, _ptr(q), None, None))
    return (a, b, q) if want_q else (a, b)


def mse(W, wdtype, fmt, group, col_dtype, sT, q, a, b) -> float:
    lib = _load()
    Win = _as_input(W, wdtype)
    M, N = Win.shape
    out = np.zeros(1, np.float64)
    a = np.ascontiguousarray(a, np.float64).copy()
    b = np.ascontiguousarray(b, np.float64).copy()
    q = np.ascontiguousarray(q, np.float64)
    _check(lib.dqo_step(_ptr(Win), WDTYPES[wdtype], M, N, FORMATS[fmt], group, WDTYPES[col_dtype], sT, 4,
                        _ptr(a), _ptr(b), _ptr(q), None, None, _ptr(out)))
    return float(out[0])


def project(kind: int, v: float) -> float:
    """Nearest admissible inverse scale (PROJ_F16 / PROJ_BF16 / PROJ_E4M3 / PROJ_E8M0)."""
    return _load().dqo_project(kind, float(v))


def encode(kind: int, v: float) -> int:
    return int(_load().dqo_encode(kind, float(v)))


def quant_index(w: float, scale: float, grid, even) -> int:
    """Index of the nearest grid value to w/scale (ties to the neighbour flagged even)."""
    g = np.ascontiguousarray(grid, np.float64)
    e = np.ascontiguousarray(even, np.uint8)
    return int(_load().dqo_quant_index(float(w), float(scale), _ptr(g), _ptr(e), len(g)))


def quant_value(fmt: str, w: float, ab: float) -> float:
    return float(_load().dqo_quant_value(FORMATS[fmt], float(w), float(ab)))


def absmax_scale(w, qmax: float) -> float:
    x = np.ascontiguousarray(w, np.float64)
    return float(_load().dqo_absmax_scale(_ptr(x), len(x), float(qmax)))


def num_threads() -> int:
    return int(_load().dqo_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of the oracle's later parallel loops (e.g. 1 to time it on one core)."""
    _load().dqo_set_num_threads(int(n))
