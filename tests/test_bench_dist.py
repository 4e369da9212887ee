"""The multi-process host logic of bench.py on CPU: world size 2 over gloo
(127.0.0.1).  Replicas only: the timing reduction is a max over ranks, the
reference arm runs on rank 0 alone."""

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


def _env(rank: int, world: int, port: int):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)


def _max_worker(rank: int, world: int, port: int, out_dir: str):
    _env(rank, world, port)
    import torch
    import torch.distributed as dist

    import bench

    bench.init_dist(world, "gloo")
    got = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
    bench.barrier(world)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
        f.write(repr(got))


def _reference_worker(rank: int, world: int, port: int, out_dir: str):
    _env(rank, world, port)
    import contextlib
    import io

    import bench

    bench.oracle_step_times = lambda w: (0.25, 0.5)  # stands in for the oracle's timing
    args = type("A", (), {"steps": 2, "warmup": 1, "impl": "reference"})()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args)
    with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
        f.write(buf.getvalue())


def test_max_over_ranks_gloo(tmp_path):
    mp.spawn(_max_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        assert float((tmp_path / f"r{r}.txt").read_text()) == pytest.approx(2.5)


def test_reference_arm_prints_on_rank0_only(tmp_path):
    mp.spawn(_reference_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    lines = [ln for ln in (tmp_path / "r0.txt").read_text().splitlines() if ln.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["extrapolated_ms_per_full_step"] == pytest.approx(500.0)
    assert rec["ms_per_step"] < 250.0  # the wall time it ran, not the stand-in figure
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
    assert (tmp_path / "r1.txt").read_text() == ""
