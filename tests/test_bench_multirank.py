"""Multi-rank host logic of bench.py on CPU: two gloo ranks (no GPU).

The bench shards the work as independent batches per rank (weak scaling, no
data-path collective); the only cross-rank operations are the barrier and the
MAX reduction of each rank's device time. These run here over gloo exactly as
they run over NCCL on GPUs.
"""
from __future__ import annotations

import argparse
import contextlib
import io
import json
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    from sliding_window_sigmoid_b200 import inputs

    w, r, _ = bench.dist_setup()
    assert (w, r) == (world, rank) and dist.get_backend() == "gloo"
    res = {}
    # MAX over ranks of each rank's own time
    res["max"] = bench.max_over_ranks(1.5 * (rank + 1), world)
    bench.barrier(world)
    # each rank draws its own batch: the inputs differ across ranks
    q = inputs.qkv(1, 8, 2, 1, 4, seed=bench.rank_seed(rank))[0]
    got = [None] * world
    dist.all_gather_object(got, q.float().sum().item())
    res["sums"] = got
    # whole-job value: units of all ranks over the slowest rank's time
    res["value"] = bench.job_value(1e12, world, 4, res["max"] * 1e3)
    # the reference arm: rank 0 alone runs and prints; the others exit without work
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(argparse.Namespace(steps=1, warmup=0))
    res["ref_out"] = buf.getvalue()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_two_gloo_ranks_max_seeds_value_and_reference_arm(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["max"] == pytest.approx(3.0)                 # slowest of 1.5 and 3.0
        assert r["value"] == pytest.approx(1e12 * 2 * 4 / 3.0 / 1e12)
        assert r["sums"][0] != r["sums"][1]                   # independent batches
    line = json.loads(res[0]["ref_out"].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == world and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert res[1]["ref_out"] == ""


def test_bwd_traffic_from_captures_and_source_hash(tmp_path, monkeypatch):
    """`traffic` of the backward call: the DRAM bytes of the committed batch-4
    captures (both kernels) scaled to the batch, and None once the kernel
    source differs from the captured one."""
    import re
    import shutil
    import sys
    sys.path.insert(0, ROOT)
    import bench
    want = 0.0
    for role in ("dq", "dkdv"):
        with open(os.path.join(ROOT, "profiles", f"swat_bwd_tc_{role}_d64_sigmoid_B4.md")) as f:
            text = f.read()
        for kind in ("read", "write"):
            want += float(re.search(r"dram__bytes_%s\.sum \| ([0-9.]+) Mbyte" % kind, text).group(1)) * 1e6
    assert bench.bwd_traffic_per_call(4) == pytest.approx(want)
    assert bench.bwd_traffic_per_call(8) == pytest.approx(2 * want)
    # a copy of the tree whose kernel source changed: no traffic figure
    (tmp_path / "profiles").mkdir()
    for role in ("dq", "dkdv"):
        name = f"swat_bwd_tc_{role}_d64_sigmoid_B4.md"
        shutil.copy(os.path.join(ROOT, "profiles", name), tmp_path / "profiles" / name)
    csrc = tmp_path / "sliding_window_sigmoid_b200" / "csrc"
    csrc.mkdir(parents=True)
    src = os.path.join(ROOT, "sliding_window_sigmoid_b200", "csrc", "bwd_tc.cuh")
    shutil.copy(src, csrc / "bwd_tc.cuh")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.bwd_traffic_per_call(8) == pytest.approx(2 * want)
    with open(csrc / "bwd_tc.cuh", "a") as f:
        f.write("\n// changed\n")
    assert bench.bwd_traffic_per_call(8) is None
