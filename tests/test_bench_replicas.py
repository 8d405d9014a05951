"""The multi-GPU path of bench.py (replicas only) on CPU: world_size 2 under
gloo. The timing a rank reports is the max over ranks; the job's value counts
every rank's units over that time; the reference arm runs on rank 0 alone."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        ms = 1.0 + rank                              # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, world)
        out[rank] = (ms_max, bench.replica_value(16 * 16, world, ms_max))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_value_gloo_world2():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        ms_max, value = out[rank]
        assert ms_max == 2.0                          # every rank sees the slowest rank's time
        assert value == pytest.approx(16 * 16 * world / 2e-3)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_value(100, 1, 10.0) == pytest.approx(1e4)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    a = bench.parse()
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(a)
    assert buf.getvalue() == ""                       # the other ranks exit without work


def test_reference_arm_line_on_rank_zero(monkeypatch):
    # the oracle on a tiny stand-in shape, so the test stays fast: the line
    # must carry the contract's keys, with the oracle as the CPU baseline and
    # an e2e that moves no bytes
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setitem(bench.SHAPES, "olmoe", (256, 128, 4, 2))
    monkeypatch.setattr(bench, "H", 256)
    monkeypatch.setattr(bench, "I", 128)
    monkeypatch.setattr(bench, "E", 4)
    monkeypatch.setattr(bench, "K", 2)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3", "--T", "4"])
    a = bench.parse()
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(a)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "layer-tokens/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["higher_is_better"] is True and line["steps"] == 1 and line["warmup"] == 3
