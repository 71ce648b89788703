"""The multi-process plumbing of bench.py on the CPU (gloo, world size 2):
replicas only, so the only collectives are the barrier and the maximum of
the per-rank timings; rank 0 alone prints."""
import io
import json
import os
import socket
import sys
import types
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        m = bench.max_over_ranks(1.5 + rank, world)
        bench.barrier(world)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"max": m}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    for r in range(world):
        with open(tmp_path / f"r{r}.json") as f:
            assert json.load(f)["max"] == 2.5


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, 1) == 3.25
    bench.barrier(1)


def test_gpus_flag_must_match_world_size(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    with pytest.raises(SystemExit):
        bench.dist_setup(2)


def test_reference_arm_prints_on_rank0_only():
    """Under torchrun every rank runs --impl reference; ranks other than 0
    return without work or output."""
    args = types.SimpleNamespace(steps=1, warmup=0, gpus=2)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args, rank=1, world=2)
    assert buf.getvalue() == ""
