"""Helpers for the GPU parity tests: decode library outputs into the values the oracle reports."""
from __future__ import annotations

import numpy as np
import torch


def block_scale_values(fmt: str, t: torch.Tensor) -> np.ndarray:
    """Stored block-scale factor values (fp16 value, 2^k, or E4M3 value e)."""
    t = t.cpu()
    if fmt == "int4":
        return t.to(torch.float64).numpy()
    if fmt == "mxint4":
        return np.ldexp(1.0, t.numpy().astype(np.int64) - 127)
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def col_scale_values(t: torch.Tensor) -> np.ndarray:
    return t.cpu().to(torch.float64).numpy()


def identity_mse_tolerance(sum_w2_over_mn: float, mse: np.ndarray, group: int) -> np.ndarray:
    """Error bound of the per-iteration MSE taken from the block sums.

    mse[t] for t < T comes from sum W^2 - sum_blocks (2 a num - a^2 den) with num
    and den fp32 sums of at most 8 + log2(G/8) roundings each; so the absolute
    error is at most 2 * (8 + log2(G/8)) * 2^-24 * (2 a num + a^2 den) summed over
    the blocks, i.e. about 4 * (8 + log2(G/8)) * 2^-24 * sum W^2.  The final MSE is
    computed directly in fp64 and held to the plain tolerance."""
    levels = 8 + int(np.log2(max(group // 8, 1)))
    return 4.0 * levels * 2.0 ** -24 * sum_w2_over_mn / np.maximum(mse, 1e-300)


def compare_with_oracle(fmt: str, gpu: dict, orc: dict, mse_rtol: float = 1e-4, label: str = "",
                        sum_w2_over_mn: float = None, group: int = 64):
    """Bit-exact codes and scales; final MSE within mse_rtol relative (spec tolerance);
    earlier MSE entries within mse_rtol or the identity's error bound, whichever is larger."""
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
    np.testing.assert_allclose(mse[-1], orc["mse"][-1], rtol=mse_rtol, atol=0, err_msg=label + " final mse")
    if len(mse) > 1:
        tol = np.full(len(mse) - 1, mse_rtol)
        if sum_w2_over_mn is not None:
            tol = np.maximum(tol, identity_mse_tolerance(sum_w2_over_mn, orc["mse"][:-1], group))
        rel = np.abs(mse[:-1] - orc["mse"][:-1]) / np.maximum(np.abs(orc["mse"][:-1]), 1e-300)
        both_zero = (mse[:-1] == 0) & (orc["mse"][:-1] == 0)
        assert np.all((rel <= tol) | both_zero), (label, rel, tol)
