"""Helpers for the GPU parity tests: decode library outputs into the values the oracle reports."""
from __future__ import annotations

import numpy as np
import torch


def block_scale_values(fmt: str, t: torch.Tensor) -> np.ndarray:
    """Stored block-scale factor values (fp16 value, 2^k, or E4M3 value e)."""
    t = t.cpu()
    if fmt == "int4":
        return t.to(torch.float64).numpy()
    if fmt in ("mxint4", "mxfp4", "mxint8", "mxfp8"):
        return np.ldexp(1.0, t.numpy().astype(np.int64) - 127)
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def col_scale_values(t: torch.Tensor) -> np.ndarray:
    return t.cpu().to(torch.float64).numpy()


def compare_with_oracle(fmt: str, gpu: dict, orc: dict, mse_rtol: float = 1e-4, label: str = ""):
    """Bit-exact codes and scales; every per-iteration MSE within mse_rtol relative (spec tolerance)."""
    codes = gpu["codes"].cpu().numpy()
    a = block_scale_values(fmt, gpu["block_scales"])
    b = col_scale_values(gpu["col_scales"])
    mse = gpu["mse"].cpu().numpy()
    bad_a = np.argwhere(a != orc["a"])
    assert bad_a.size == 0, "%s block scales differ at %d places, first %s: gpu %r oracle %r" % (
        label, len(bad_a), bad_a[:3].tolist(), a[tuple(bad_a[0])], orc["a"][tuple(bad_a[0])])
    bad_b = np.nonzero(b != orc["b"])[0]
    assert bad_b.size == 0, "%s col scales differ at %d cols, first %s: gpu %r oracle %r" % (
        label, len(bad_b), bad_b[:3].tolist(), b[bad_b[0]], orc["b"][bad_b[0]])
    if fmt == "nvfp4":
        assert float(gpu["tensor_scale"].cpu()[0]) == orc["sT"]
    bad_c = np.argwhere(codes != orc["codes"])
    assert bad_c.size == 0, "%s codes differ at %d bytes, first %s" % (label, len(bad_c), bad_c[:3].tolist())
    np.testing.assert_allclose(mse, orc["mse"], rtol=mse_rtol, atol=0, err_msg=label + " mse")
