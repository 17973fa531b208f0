"""CPU-side checks of the C ABI library and the host logic of the binding (no GPU)."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

from calibration_free_weight_dualquant_b200 import binding, build, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "dq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dq_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib_path():
    return build.build()


def test_library_exports_every_declared_symbol(lib_path):
    names = declared_symbols()
    assert {"dq_rtn", "dq_solve", "dq_workspace_bytes", "dq_sync_status", "dq_status_str"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (dq_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(lib_path)
    for n in names:
        assert hasattr(lib, n)


def test_status_strings(lib_path):
    lib = ctypes.CDLL(lib_path)
    lib.dq_status_str.restype = ctypes.c_char_p
    for code, name in binding.STATUS.items():
        assert lib.dq_status_str(code).decode().startswith(name)
    assert b"unknown" in lib.dq_status_str(99)


def test_output_sizes_storage_pin():
    """DualQuant App. I / Table 12: 224 linears at INT4-G64 -> 3.49 GB codes + 0.22 GB fp16 scales."""
    tot_codes = tot_scales = 0
    for _ in range(synth.LLAMA31_8B_LAYERS):
        for _, r, c in synth.LLAMA31_8B_LAYER:
            n = binding.output_nbytes(r, c, "int4", 64, "f16")
            tot_codes += n["codes"]
            tot_scales += n["block_scales"]
    assert "%.2f" % (tot_codes / 1e9) == "3.49"
    assert "%.2f" % (tot_scales / 1e9) == "0.22"
    n = binding.output_nbytes(4096, 4096, "nvfp4")
    assert n["block_scales"] == 4096 * 256 and n["tensor_scale"] == 4
    n = binding.output_nbytes(4096, 14336, "mxint4")
    assert n["block_scales"] == 4096 * 448 and n["col_scales"] == 14336 * 2


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(binding.DQError):
        binding.load_library()


def test_format_numbering_matches_header():
    """The binding's format numbers are the header's dq_format values, and the oracle's format names
    cover every one of them (their numbers mirror the header's by value only)."""
    import oracle
    text = open(os.path.join(ROOT, "include", "dq.h")).read()
    body = re.search(r"typedef enum \{([^}]*)\} dq_format;", text).group(1)
    header = {k: int(v) for k, v in re.findall(r"DQ_(\w+)\s*=\s*(\d+)", body)}
    assert header == {f.name: int(f) for f in binding.Format}
    assert set(oracle.FORMATS) == {f.name.lower() for f in binding.Format}


def test_byte_code_formats_output_sizes():
    """MXINT8 and MXFP8 store one byte per code; the 4-bit formats two codes per byte."""
    for fmt in ("mxint8", "mxfp8"):
        n = binding.output_nbytes(4096, 14336, fmt)
        assert n["codes"] == 4096 * 14336 and n["block_scales"] == 4096 * 448 and n["tensor_scale"] == 0
    for fmt in ("int4", "mxint4", "nvfp4", "mxfp4"):
        assert binding.output_nbytes(64, 512, fmt)["codes"] == 64 * 256
    out = binding.alloc_outputs(8, 64, "mxfp8", 32, "bf16", 2, "cpu")
    assert tuple(out["codes"].shape) == (8, 64)


def test_host_side_argument_checks_for_the_8bit_formats(lib_path):
    """Rejected on the host before any device work (so no GPU is needed here): the MX 8-bit formats
    take group 32 only, the activation quantizer writes 4-bit codes only, and the byte codes must be
    8-byte aligned."""
    lib = binding.load_library()
    bufs = [ctypes.create_string_buffer(4096 + 64) for _ in range(5)]
    base = [((ctypes.addressof(b) + 63) // 64) * 64 for b in bufs]
    W = base[0]
    wsbuf = ctypes.create_string_buffer(1024)
    ws = ((ctypes.addressof(wsbuf) + 255) // 256) * 256

    def outs(codes_off=0):
        return binding._Outputs(base[1] + codes_off, base[2], base[3], base[4], base[4] + 1024)

    for fmt in (int(binding.Format.MXINT8), int(binding.Format.MXFP8)):
        for g, want in ((16, 2), (64, 2)):
            o = outs()
            assert lib.dq_solve(W, 1, 4, 64, fmt, g, 2, 1, ctypes.byref(o), None, 0, None) == want
        # byte codes 4-byte aligned only: DQ_EINVAL; 8-byte aligned they pass the output checks and stop
        # later (no device here: DQ_ECUDA; with one, the empty workspace: DQ_EWORKSPACE)
        o = outs(codes_off=4)
        assert lib.dq_solve(W, 1, 4, 64, fmt, 32, 2, 1, ctypes.byref(o), ws, 0, None) == 1
        o = outs(codes_off=8)
        assert lib.dq_solve(W, 1, 4, 64, fmt, 32, 2, 1, ctypes.byref(o), ws, 0, None) in (3, 5)
        o = outs()
        assert lib.dq_act_quant(W, 1, 4, 64, base[4], 1, fmt, 32, ctypes.byref(o), None, 0, None) == 2
    o = outs()
    assert lib.dq_solve(W, 1, 4, 64, 6, 32, 2, 1, ctypes.byref(o), None, 0, None) == 1   # no format 6


def test_int4_groups_are_powers_of_two(lib_path):
    """INT4 takes the power-of-two groups 8 .. 256 (a block row spans group/8 lanes of a warp); an even
    divisor of cols that is not a power of two is DQ_EUNSUPPORTED in the solver and the activation
    quantizer, decided on the host before any device work."""
    lib = binding.load_library()
    bufs = [ctypes.create_string_buffer(8192 + 64) for _ in range(5)]
    base = [((ctypes.addressof(b) + 63) // 64) * 64 for b in bufs]
    o = binding._Outputs(base[1], base[2], base[3], base[4], base[4] + 1024)
    for g in (24, 48, 96):
        cols = 2 * 96  # a multiple of every group tried
        assert lib.dq_solve(base[0], 1, 4, cols, int(binding.Format.INT4), g, 2, 2, ctypes.byref(o), None, 0,
                            None) == 2, g
        assert lib.dq_act_quant(base[0], 1, 4, cols, base[4], 1, int(binding.Format.INT4), g, ctypes.byref(o),
                                None, 0, None) == 2, g
    for g in (4, 512):
        assert lib.dq_solve(base[0], 1, 4, 1024, int(binding.Format.INT4), g, 2, 2, ctypes.byref(o), None, 0,
                            None) == 2, g


def test_act_quant_host_side_checks(lib_path):
    """dq_act_quant's argument checks, decided on the host before any device work: X 16-byte aligned,
    bf16/fp16 X and column scales, a group the format takes, codes 4-byte aligned, a workspace of
    DQ_ACT_WORKSPACE_BYTES."""
    lib = binding.load_library()
    bufs = [ctypes.create_string_buffer(8192 + 64) for _ in range(5)]
    base = [((ctypes.addressof(b) + 63) // 64) * 64 for b in bufs]
    wsbuf = ctypes.create_string_buffer(1024)
    ws = ((ctypes.addressof(wsbuf) + 255) // 256) * 256
    o = binding._Outputs(base[1], base[2], base[3], base[4], base[4] + 1024)
    I4, MX4, NV = int(binding.Format.INT4), int(binding.Format.MXINT4), int(binding.Format.NVFP4)
    act = lib.dq_act_quant
    assert act(base[0] + 8, 1, 4, 64, base[4], 1, I4, 64, ctypes.byref(o), ws, 256, None) == 1   # X not 16-byte aligned
    assert act(base[0], 0, 4, 64, base[4], 1, I4, 64, ctypes.byref(o), ws, 256, None) == 2       # fp32 X
    assert act(base[0], 1, 4, 64, base[4], 0, I4, 64, ctypes.byref(o), ws, 256, None) == 2       # fp32 column scales
    assert act(base[0], 1, 4, 64, base[4], 1, MX4, 16, ctypes.byref(o), ws, 256, None) == 2      # MXINT4 takes 32
    assert act(base[0], 1, 4, 64, base[4], 1, NV, 32, ctypes.byref(o), ws, 256, None) == 2       # NVFP4 takes 16
    assert act(base[0], 1, 4, 48, base[4], 1, I4, 32, ctypes.byref(o), ws, 256, None) == 1       # cols % group
    assert act(base[0], 1, 0, 64, base[4], 1, I4, 64, ctypes.byref(o), ws, 256, None) == 1       # no rows
    bad = binding._Outputs(base[1] + 2, base[2], base[3], base[4], base[4] + 1024)
    assert act(base[0], 1, 4, 64, base[4], 1, I4, 64, ctypes.byref(bad), ws, 256, None) == 1     # codes 2-byte aligned
    assert act(base[0], 1, 4, 64, base[4], 1, I4, 64, ctypes.byref(o), ws, 128, None) == 3       # short workspace
