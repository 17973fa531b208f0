"""Thin ctypes binding of ``libdq.so`` (C ABI in ``include/dq.h``).

Argument marshalling only: torch supplies device memory and the current
stream; every step of the solver runs in the library's CUDA kernels.  There is
no CPU fallback -- without the built library or a CUDA device every call
raises :class:`DQError`.
"""
from __future__ import annotations

import ctypes
import enum
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libdq.so")

STATUS = {0: "DQ_OK", 1: "DQ_EINVAL", 2: "DQ_EUNSUPPORTED", 3: "DQ_EWORKSPACE", 4: "DQ_ENONFINITE", 5: "DQ_ECUDA"}


class Format(enum.IntEnum):
    INT4 = 0
    MXINT4 = 1
    NVFP4 = 2
    MXFP4 = 3
    MXINT8 = 4
    MXFP8 = 5


_FMT_NAMES = {"int4": Format.INT4, "mxint4": Format.MXINT4, "nvfp4": Format.NVFP4, "mxfp4": Format.MXFP4,
              "mxint8": Format.MXINT8, "mxfp8": Format.MXFP8}
_DTYPES = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}
_COL_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}
DEFAULT_GROUP = {Format.INT4: 64, Format.MXINT4: 32, Format.NVFP4: 16, Format.MXFP4: 32, Format.MXINT8: 32,
                 Format.MXFP8: 32}
DEFAULT_COL_DTYPE = {Format.INT4: "f16", Format.MXINT4: "bf16", Format.NVFP4: "bf16", Format.MXFP4: "bf16",
                     Format.MXINT8: "bf16", Format.MXFP8: "bf16"}


def code_cols(cols: int, fmt) -> int:
    """Bytes of codes per row: one per element on the INT8 and E4M3 grids, two nibbles per byte otherwise."""
    return cols if _fmt(fmt) in (Format.MXINT8, Format.MXFP8) else cols // 2


class DQError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__("%s%s" % (STATUS.get(status, "status %d" % status), (" in " + where) if where else ""))


class _Outputs(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("block_scales", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p),
                ("col_scales", ctypes.c_void_p), ("mse", ctypes.c_void_p)]


class _Options(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("init", ctypes.c_int), ("code_changes", ctypes.c_void_p),
                ("full_passes", ctypes.c_int)]


class _Matrix(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("w_dtype", ctypes.c_int), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("out", _Outputs)]


_lib = None


def load_library():
    """Load libdq.so (built in-tree by ``build.py``); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise DQError(5, "load_library: %s is not built (run __graft_entry__.build())" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    I64, I, SZ, P = ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
    lib.dq_workspace_bytes.argtypes = [I64, I64, I, I]
    lib.dq_workspace_bytes.restype = SZ
    lib.dq_rtn.argtypes = [P, I, I64, I64, I, I, I, ctypes.POINTER(_Outputs), P, SZ, P]
    lib.dq_rtn.restype = I
    lib.dq_solve.argtypes = [P, I, I64, I64, I, I, I, I, ctypes.POINTER(_Outputs), P, SZ, P]
    lib.dq_solve.restype = I
    lib.dq_solve_mode.argtypes = [P, I, I64, I64, I, I, I, I, I, ctypes.POINTER(_Outputs), P, SZ, P]
    lib.dq_solve_mode.restype = I
    lib.dq_workspace_bytes_ex.argtypes = [I64, I64, I, I, ctypes.POINTER(_Options)]
    lib.dq_workspace_bytes_ex.restype = SZ
    lib.dq_solve_ex.argtypes = [P, I, I64, I64, I, I, I, I, ctypes.POINTER(_Options), ctypes.POINTER(_Outputs), P,
                                SZ, P]
    lib.dq_solve_ex.restype = I
    lib.dq_sync_status.argtypes = [P, P]
    lib.dq_sync_status.restype = I
    lib.dq_host_workspace_bytes.argtypes = [I64, I64, I, I, I, I]
    lib.dq_host_workspace_bytes.restype = SZ
    lib.dq_solve_host.argtypes = [P, I, I64, I64, I, I, I, I, ctypes.POINTER(_Outputs), P, SZ, P]
    lib.dq_solve_host.restype = I
    lib.dq_diagnostics.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint64)]
    lib.dq_active_block_columns.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint64)]
    lib.dq_active_block_columns.restype = I
    lib.dq_diagnostics.restype = I
    lib.dq_wait_selftest.argtypes = [P, SZ, I, P]
    lib.dq_wait_selftest.restype = I
    lib.dq_solve_static.argtypes = [P, I, I64, I64, I, I, I, I, ctypes.POINTER(_Outputs), P, P]
    lib.dq_solve_static.restype = I
    lib.dq_solve_batched.argtypes = [ctypes.POINTER(_Matrix), I, I, I, I, I, P, P, SZ, ctypes.POINTER(I), P]
    lib.dq_solve_batched.restype = I
    lib.dq_act_quant.argtypes = [P, I, I64, I64, P, I, I, I, ctypes.POINTER(_Outputs), P, SZ, P]
    lib.dq_act_quant.restype = I
    lib.dq_status_str.argtypes = [I]
    lib.dq_status_str.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _fmt(fmt) -> Format:
    return _FMT_NAMES[fmt] if isinstance(fmt, str) else Format(fmt)


def output_nbytes(rows: int, cols: int, fmt, group: Optional[int] = None, col_dtype: Optional[str] = None) -> dict:
    """Bytes of each output: packed codes, block scales, column scales (host-side size arithmetic)."""
    f = _fmt(fmt)
    g = DEFAULT_GROUP[f] if group is None else group
    cd = DEFAULT_COL_DTYPE[f] if col_dtype is None else col_dtype
    return {"codes": rows * code_cols(cols, f), "block_scales": rows * (cols // g) * (2 if f == Format.INT4 else 1),
            "col_scales": cols * 2, "tensor_scale": 4 if f == Format.NVFP4 else 0}


def workspace_bytes(rows: int, cols: int, fmt, group: Optional[int] = None) -> int:
    f = _fmt(fmt)
    g = DEFAULT_GROUP[f] if group is None else group
    return int(load_library().dq_workspace_bytes(rows, cols, int(f), g))


def alloc_outputs(rows: int, cols: int, fmt, group: int, col_dtype: str, iters: int, device) -> dict:
    f = _fmt(fmt)
    nb = cols // group
    return {
        "codes": torch.empty((rows, code_cols(cols, f)), dtype=torch.uint8, device=device),
        "block_scales": torch.empty((rows, nb), dtype=torch.float16 if f == Format.INT4 else torch.uint8,
                                    device=device),
        "tensor_scale": torch.empty(1, dtype=torch.float32, device=device),
        "col_scales": torch.empty(cols, dtype=_COL_DTYPES[col_dtype], device=device),
        "mse": torch.empty(iters + 1, dtype=torch.float64, device=device),
    }


def _outputs_struct(out: dict) -> _Outputs:
    return _Outputs(out["codes"].data_ptr(), out["block_scales"].data_ptr(), out["tensor_scale"].data_ptr(),
                    out["col_scales"].data_ptr(), out["mse"].data_ptr())


def _stream_ptr(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


MODES = {"dual": 0, "row": 1, "col": 2}
INITS = {"rtn": 0, "l1": 1, "given": 2}


def dq_solve(W: torch.Tensor, fmt, group: Optional[int] = None, iters: int = 0, col_dtype: Optional[str] = None,
             out: Optional[dict] = None, workspace: Optional[torch.Tensor] = None, stream=None,
             check: bool = True, mode: str = "dual", init: str = "rtn", init_scales: Optional[dict] = None,
             changes: bool = False, full_passes: bool = False) -> dict:
    """Enqueue dq_solve on a CUDA tensor W [rows, cols]; returns the output tensors.

    ``check`` waits for the stream and raises on a device-reported status
    (non-finite W, inadmissible warm-start scales).  Pass preallocated ``out`` /
    ``workspace`` to avoid allocations (e.g. when timing).  ``mode``: "dual",
    "row" or "col" (dq_mode).  ``init``: "rtn", "l1" or "given" (dq_init); with
    "given" the initial scales are ``init_scales`` ({"block_scales",
    "col_scales", "tensor_scale"} in storage format, e.g. a previous call's
    outputs), copied into ``out`` first, or whatever ``out`` already holds.
    ``changes`` adds out["code_changes"] (int64 [iters+1], changed codes per
    iteration).  ``full_passes`` makes every iteration process every
    block-column (no skipping of block-columns at a fixed point; same outputs)."""
    lib = load_library()
    if not W.is_cuda:
        raise DQError(1, "dq_solve: W must be a CUDA tensor (use solve() for host tensors)")
    f = _fmt(fmt)
    g = DEFAULT_GROUP[f] if group is None else group
    cd = DEFAULT_COL_DTYPE[f] if col_dtype is None else col_dtype
    rows, cols = W.shape
    if W.dtype not in _DTYPES or not W.is_contiguous():
        raise DQError(1, "dq_solve: W must be contiguous f32/bf16/f16")
    if out is None:
        out = alloc_outputs(rows, cols, f, g, cd, iters, W.device)
    extended = init != "rtn" or changes or full_passes
    opts = None
    if extended:
        if init == "given" and init_scales is not None:
            for k in ("block_scales", "col_scales", "tensor_scale"):
                if k in init_scales:
                    out[k].view(-1).copy_(init_scales[k].reshape(-1))
        if changes:
            out["code_changes"] = torch.empty(iters + 1, dtype=torch.int64, device=W.device)
        opts = _Options(MODES[mode], INITS[init], out["code_changes"].data_ptr() if changes else None,
                        1 if full_passes else 0)
    if workspace is None:
        if extended:
            nbytes = lib.dq_workspace_bytes_ex(rows, cols, int(f), g, ctypes.byref(opts))
        else:
            nbytes = lib.dq_workspace_bytes(rows, cols, int(f), g)
        if nbytes == 0:
            raise DQError(1, "dq_workspace_bytes")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    o = _outputs_struct(out)
    cdt = 2 if cd == "f16" else 1
    if extended:
        st = lib.dq_solve_ex(W.data_ptr(), _DTYPES[W.dtype], rows, cols, int(f), g, iters, cdt, ctypes.byref(opts),
                             ctypes.byref(o), workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    elif mode == "dual":
        st = lib.dq_solve(W.data_ptr(), _DTYPES[W.dtype], rows, cols, int(f), g, iters, cdt, ctypes.byref(o),
                          workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    else:
        st = lib.dq_solve_mode(W.data_ptr(), _DTYPES[W.dtype], rows, cols, int(f), g, iters, cdt, MODES[mode],
                               ctypes.byref(o), workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    if st != 0:
        raise DQError(st, "dq_solve")
    if check:
        st = lib.dq_sync_status(workspace.data_ptr(), _stream_ptr(stream))
        if st != 0:
            raise DQError(st, "dq_solve (device)")
    out["workspace"] = workspace
    return out


def dq_solve_static(W: torch.Tensor, fmt, group: Optional[int] = None, iters: int = 0,
                    col_dtype: Optional[str] = None, out: Optional[dict] = None, status: Optional[torch.Tensor] = None,
                    stream=None, check: bool = True) -> dict:
    """Enqueue dq_solve_static: dq_solve with its scratch in the library's own
    fixed device array (no workspace).  ``status`` is an optional int32 CUDA
    tensor of one element that receives the device-side status; with ``check``
    the call waits for the stream and raises on a non-zero status.  Pass
    preallocated ``out`` and ``status`` to keep the call free of allocations."""
    lib = load_library()
    if not W.is_cuda:
        raise DQError(1, "dq_solve_static: W must be a CUDA tensor")
    f = _fmt(fmt)
    g = DEFAULT_GROUP[f] if group is None else group
    cd = DEFAULT_COL_DTYPE[f] if col_dtype is None else col_dtype
    rows, cols = W.shape
    if W.dtype not in _DTYPES or not W.is_contiguous():
        raise DQError(1, "dq_solve_static: W must be contiguous f32/bf16/f16")
    if out is None:
        out = alloc_outputs(rows, cols, f, g, cd, iters, W.device)
    if status is None and check:
        status = torch.full((1,), -1, dtype=torch.int32, device=W.device)
    if status is not None and (status.dtype != torch.int32 or not status.is_cuda):
        raise DQError(1, "dq_solve_static: status must be an int32 CUDA tensor")
    o = _outputs_struct(out)
    st = lib.dq_solve_static(W.data_ptr(), _DTYPES[W.dtype], rows, cols, int(f), g, iters, 2 if cd == "f16" else 1,
                             ctypes.byref(o), None if status is None else status.data_ptr(), _stream_ptr(stream))
    if st != 0:
        raise DQError(st, "dq_solve_static")
    if check:
        (torch.cuda.current_stream() if stream is None else stream).synchronize()
        dev_st = int(status.cpu()[0])
        if dev_st != 0:
            raise DQError(dev_st, "dq_solve_static (device)")
    out["status"] = status
    return out


def dq_solve_batched(Ws, fmt, group: Optional[int] = None, iters: int = 0, col_dtype: Optional[str] = None,
                     outs: Optional[list] = None, workspace: Optional[torch.Tensor] = None,
                     status: Optional[torch.Tensor] = None, stream=None, check: bool = True) -> list:
    """Enqueue dq_solve_batched: every CUDA matrix of ``Ws`` solved one after another on one stream with
    one shared workspace.  Returns the list of output dicts; ``check`` waits and raises on the first
    matrix whose device-side status is not DQ_OK."""
    lib = load_library()
    f = _fmt(fmt)
    g = DEFAULT_GROUP[f] if group is None else group
    cd = DEFAULT_COL_DTYPE[f] if col_dtype is None else col_dtype
    n = len(Ws)
    if n == 0:
        return []
    dev = Ws[0].device
    for W in Ws:
        if not W.is_cuda or W.dtype not in _DTYPES or not W.is_contiguous() or W.dim() != 2:
            raise DQError(1, "dq_solve_batched: every W must be a contiguous 2-D CUDA f32/bf16/f16 tensor")
    if outs is None:
        outs = [alloc_outputs(W.shape[0], W.shape[1], f, g, cd, iters, dev) for W in Ws]
    if workspace is None:
        nbytes = max(int(lib.dq_workspace_bytes(W.shape[0], W.shape[1], int(f), g)) for W in Ws)
        if nbytes == 0:
            raise DQError(1, "dq_workspace_bytes")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    if status is None:
        status = torch.full((n,), -1, dtype=torch.int32, device=dev)
    mats = (_Matrix * n)()
    for i, (W, o) in enumerate(zip(Ws, outs)):
        mats[i].W = W.data_ptr()
        mats[i].w_dtype = _DTYPES[W.dtype]
        mats[i].rows, mats[i].cols = W.shape
        mats[i].out = _outputs_struct(o)
    bad = ctypes.c_int(-1)
    st = lib.dq_solve_batched(mats, n, int(f), g, iters, 2 if cd == "f16" else 1, status.data_ptr(),
                              workspace.data_ptr(), workspace.numel(), ctypes.byref(bad), _stream_ptr(stream))
    if st != 0:
        raise DQError(st, "dq_solve_batched (matrix %d)" % bad.value)
    if check:
        (torch.cuda.current_stream() if stream is None else stream).synchronize()
        sts = status.cpu().tolist()
        for i, v in enumerate(sts):
            if v != 0:
                raise DQError(v, "dq_solve_batched (device, matrix %d)" % i)
    for o in outs:
        o["workspace"] = workspace
    return outs


ACT_WORKSPACE_BYTES = 256


def dq_act_quant(X: torch.Tensor, col_scales: torch.Tensor, fmt, group: Optional[int] = None,
                 out: Optional[dict] = None, workspace: Optional[torch.Tensor] = None, stream=None,
                 check: bool = True) -> dict:
    """Enqueue dq_act_quant: X [tokens, cols] (bf16/f16 CUDA) times the column inverse scales, quantized
    row-wise in the format (codes, group scales, NVFP4 tensor scale)."""
    lib = load_library()
    f = _fmt(fmt)
    g = DEFAULT_GROUP[f] if group is None else group
    if not X.is_cuda or X.dtype not in (torch.bfloat16, torch.float16) or not X.is_contiguous() or X.dim() != 2:
        raise DQError(1, "dq_act_quant: X must be a contiguous 2-D bf16/f16 CUDA tensor")
    if col_scales.dtype not in (torch.bfloat16, torch.float16) or not col_scales.is_cuda:
        raise DQError(1, "dq_act_quant: col_scales must be a bf16/f16 CUDA tensor")
    rows, cols = X.shape
    if out is None:
        out = {"codes": torch.empty((rows, cols // 2), dtype=torch.uint8, device=X.device),
               "block_scales": torch.empty((rows, cols // g), dtype=torch.float16 if f == Format.INT4 else torch.uint8,
                                           device=X.device),
               "tensor_scale": torch.empty(1, dtype=torch.float32, device=X.device)}
    if workspace is None:
        workspace = torch.empty(ACT_WORKSPACE_BYTES, dtype=torch.uint8, device=X.device)
    o = _Outputs(out["codes"].data_ptr(), out["block_scales"].data_ptr(), out["tensor_scale"].data_ptr(), None, None)
    st = lib.dq_act_quant(X.data_ptr(), _DTYPES[X.dtype], rows, cols, col_scales.data_ptr(),
                          _DTYPES[col_scales.dtype], int(f), g, ctypes.byref(o), workspace.data_ptr(),
                          workspace.numel(), _stream_ptr(stream))
    if st != 0:
        raise DQError(st, "dq_act_quant")
    if check:
        st = lib.dq_sync_status(workspace.data_ptr(), _stream_ptr(stream))
        if st != 0:
            raise DQError(st, "dq_act_quant (device)")
    out["workspace"] = workspace
    return out


def dq_rtn(W: torch.Tensor, fmt, group: Optional[int] = None, col_dtype: Optional[str] = None, **kw) -> dict:
    """Absmax RTN (beta = 1) through the library's dq_rtn entry point."""
    lib = load_library()
    f = _fmt(fmt)
    g = DEFAULT_GROUP[f] if group is None else group
    cd = DEFAULT_COL_DTYPE[f] if col_dtype is None else col_dtype
    rows, cols = W.shape
    out = kw.get("out") or alloc_outputs(rows, cols, f, g, cd, 0, W.device)
    ws = kw.get("workspace")
    if ws is None:
        ws = torch.empty(lib.dq_workspace_bytes(rows, cols, int(f), g), dtype=torch.uint8, device=W.device)
    o = _outputs_struct(out)
    stream = kw.get("stream")
    st = lib.dq_rtn(W.data_ptr(), _DTYPES[W.dtype], rows, cols, int(f), g, 2 if cd == "f16" else 1, ctypes.byref(o),
                    ws.data_ptr(), ws.numel(), _stream_ptr(stream))
    if st != 0:
        raise DQError(st, "dq_rtn")
    st = lib.dq_sync_status(ws.data_ptr(), _stream_ptr(stream))
    if st != 0:
        raise DQError(st, "dq_rtn (device)")
    return out


def host_workspace_bytes(rows: int, cols: int, w_dtype: torch.dtype, fmt, group: int, iters: int) -> int:
    return int(load_library().dq_host_workspace_bytes(rows, cols, _DTYPES[w_dtype], int(_fmt(fmt)), group, iters))


def solve(W: torch.Tensor, fmt="nvfp4", group: Optional[int] = None, iters: int = 15,
          col_dtype: Optional[str] = None, out: Optional[dict] = None, device_workspace: Optional[torch.Tensor] = None,
          stream=None) -> dict:
    """User-level solve.  A host (CPU) W goes through ``dq_solve_host``: the copy
    to the device, the solve and the copy of the outputs back all happen inside
    the library call, and host output tensors are returned.  A CUDA W goes
    through ``dq_solve``."""
    f = _fmt(fmt)
    g = DEFAULT_GROUP[f] if group is None else group
    cd = DEFAULT_COL_DTYPE[f] if col_dtype is None else col_dtype
    if W.is_cuda:
        return dq_solve(W, f, g, iters, cd, out=out, stream=stream)
    lib = load_library()
    rows, cols = W.shape
    if W.dtype not in _DTYPES or not W.is_contiguous():
        raise DQError(1, "solve: W must be contiguous f32/bf16/f16")
    if out is None:
        out = alloc_outputs(rows, cols, f, g, cd, iters, "cpu")
    if device_workspace is None:
        nbytes = lib.dq_host_workspace_bytes(rows, cols, _DTYPES[W.dtype], int(f), g, iters)
        if nbytes == 0:
            raise DQError(1, "dq_host_workspace_bytes")
        device_workspace = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    o = _outputs_struct(out)
    st = lib.dq_solve_host(W.data_ptr(), _DTYPES[W.dtype], rows, cols, int(f), g, iters, 2 if cd == "f16" else 1,
                           ctypes.byref(o), device_workspace.data_ptr(), device_workspace.numel(),
                           _stream_ptr(stream))
    if st != 0:
        raise DQError(st, "dq_solve_host")
    return out


def rtn(W: torch.Tensor, fmt="nvfp4", group: Optional[int] = None, col_dtype: Optional[str] = None) -> dict:
    """User-level absmax RTN (the 0-iteration solve)."""
    return solve(W, fmt, group, 0, col_dtype)


def wait_selftest(workspace: torch.Tensor, which: int = 0, stream=None) -> int:
    """Run the library's bounded-wait self-test on ``workspace`` (device, >= 512 bytes) and return the
    device status it leaves (dq_sync_status): DQ_ECUDA (5) when the wait gave up as it should.
    ``which``: 0 waits on a pending count in global memory, 1 on a shared-memory ring barrier."""
    lib = load_library()
    st = lib.dq_wait_selftest(workspace.data_ptr(), workspace.numel(), int(which), _stream_ptr(stream))
    if st != 0:
        raise DQError(st, "dq_wait_selftest")
    return lib.dq_sync_status(workspace.data_ptr(), _stream_ptr(stream))


def diagnostics(workspace: torch.Tensor, stream=None) -> dict:
    """Exact-path counters of the last solve that used this workspace."""
    lib = load_library()
    arr = (ctypes.c_uint64 * 4)()
    st = lib.dq_diagnostics(workspace.data_ptr(), _stream_ptr(stream), arr)
    if st != 0:
        raise DQError(st, "dq_diagnostics")
    return {"quant_exact_lane_rows": int(arr[0]), "block_exact": int(arr[1]), "col_exact": int(arr[2]),
            "quant_tie_lane_rows": int(arr[3])}


def active_block_columns(workspace: torch.Tensor, stream=None) -> int:
    """Block-columns the BCD iterations of the last solve on this workspace processed, summed over the
    iterations (iters * cols/group when none reached a fixed point early)."""
    lib = load_library()
    out = ctypes.c_uint64(0)
    st = lib.dq_active_block_columns(workspace.data_ptr(), _stream_ptr(stream), ctypes.byref(out))
    if st != 0:
        raise DQError(st, "dq_active_block_columns")
    return int(out.value)
