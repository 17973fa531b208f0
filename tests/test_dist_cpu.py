"""The multi-process (N > 1) plumbing of bench.py on CPU: two ranks over gloo on 127.0.0.1.

Each rank of a multi-GPU run solves its own replica (no data-path collective);
the ranks meet only in barriers and in the max over ranks of the timed region.
These tests run that plumbing, and the oracle arm under two ranks (rank 0 alone
runs and prints; rank 1 exits without work), as spawned processes.
"""
from __future__ import annotations

import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, outdir: str):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench
    from calibration_free_weight_dualquant_b200 import synth
    r, w, _, dist = bench.dist_setup(world)
    assert (r, w) == (rank, world)
    assert dist.get_backend() == "gloo"
    mx = bench.max_over_ranks(float(rank + 1) * 1.5, dist)
    bench.barrier(dist)

    class Args:
        steps, warmup, gpus, ref_rows = 1, 0, world, 8

    out = os.path.join(outdir, "rank%d.txt" % rank)
    with open(out, "w") as f:
        old = sys.stdout
        sys.stdout = f
        try:
            bench.run_reference(Args, synth.WORKLOADS["int4_g64_256x512_f32"], r, w, dist)
        finally:
            sys.stdout = old
    with open(os.path.join(outdir, "max%d.txt" % rank), "w") as f:
        f.write(repr(mx))
    bench.barrier(dist)
    dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_ranks_over_gloo(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn")
    for rank in (0, 1):
        assert float((tmp_path / ("max%d.txt" % rank)).read_text()) == 3.0  # the max over both ranks
    line0 = (tmp_path / "rank0.txt").read_text().strip()
    assert (tmp_path / "rank1.txt").read_text().strip() == ""  # only rank 0 runs the oracle arm
    d = json.loads(line0)
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["config"]["parallelism"] == "replicas x2"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
