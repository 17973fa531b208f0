"""Host-side arithmetic of bench.py (no GPU): the algorithmic bytes the roofline divides by, and the
gating of the ncu traffic figure on the kernel sources it was taken of."""
from __future__ import annotations

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from calibration_free_weight_dualquant_b200 import synth  # noqa: E402


def test_algorithmic_bytes_per_iteration():
    """One BCD iteration reads W once and reads and writes the block scales and the column scales."""
    nv = synth.WORKLOADS["nvfp4_g16_gateup_14336x4096"]
    # W 14336 x 4096 bf16, E4M3 block scales 14336 x 256 (1 byte) read and written, bf16 b read and written
    assert bench.algorithmic_bytes_per_iter(nv) == 14336 * 4096 * 2 + 2 * 14336 * 256 + 2 * 4096 * 2 == 124796928
    mx = synth.WORKLOADS["mxint4_g32_downproj_4096x14336"]
    assert bench.algorithmic_bytes_per_iter(mx) == 4096 * 14336 * 2 + 2 * 4096 * 448 + 2 * 14336 * 2 == 121167872
    i4 = synth.WORKLOADS["int4_g64_qproj_4096x4096"]
    # fp16 block scales: 2 bytes each
    assert bench.algorithmic_bytes_per_iter(i4) == 4096 * 4096 * 2 + 2 * 4096 * 64 * 2 + 2 * 4096 * 2
    f32 = synth.WORKLOADS["int4_g64_256x512_f32"]
    assert bench.algorithmic_bytes_per_iter(f32) == 256 * 512 * 4 + 2 * 256 * 8 * 2 + 2 * 512 * 2


def test_traffic_is_reported_only_for_the_profiled_kernel(tmp_path, monkeypatch):
    """The committed DRAM figure is used while the kernel sources hash as when it was captured."""
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_hash", lambda: "abc123")
    (prof / "k_iter_w.json").write_text(json.dumps({"kernel_hash": "abc123", "dram_bytes_per_pass": 42}))
    assert bench.profile_traffic("w") == 42
    (prof / "k_iter_w.json").write_text(json.dumps({"kernel_hash": "other", "dram_bytes_per_pass": 42}))
    assert bench.profile_traffic("w") is None
    assert bench.profile_traffic("missing") is None

