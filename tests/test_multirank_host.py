"""The benchmark's multi-rank logic on CPU: two ranks over gloo, as torchrun
would start them (RANK / WORLD_SIZE / LOCAL_RANK in the environment).

The GPU path shards nothing (every rank runs its own batch of the same
workload), so the only cross-rank step is the max over ranks of the timed
device time and the whole-job throughput derived from it.
"""
import contextlib
import io
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, local = bench.rank_env()
        own_ms = 100.0 + 37.5 * rank                  # the slower rank decides the job time
        max_ms = bench.max_over_ranks(own_ms, w, "cpu")
        tops = bench.job_tops(w, 4.0e11, 20, max_ms)
        # the reference arm prints only on rank 0
        buf = io.StringIO()
        if r != 0:
            with contextlib.redirect_stdout(buf):
                bench.run_reference(None, r)
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{r} {w} {local} {max_ms!r} {tops!r} {len(buf.getvalue())}\n")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_and_report_the_whole_job(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    rows = []
    for rank in range(world):
        r, w, local, max_ms, tops, printed = open(tmp_path / f"rank{rank}.txt").read().split()
        rows.append((int(r), int(w), int(local), float(max_ms), float(tops), int(printed)))
    assert [row[0] for row in rows] == [0, 1] and all(row[1] == world for row in rows)
    assert all(row[2] == row[0] for row in rows)
    assert all(row[3] == 137.5 for row in rows)          # max over ranks, on every rank
    expect = world * 4.0e11 * 20 / 0.1375 / 1e12
    assert all(row[4] == pytest.approx(expect, rel=1e-12) for row in rows)
    assert rows[1][5] == 0                                # rank 1 printed nothing


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, 1, "cpu") == 12.5
    assert bench.job_tops(1, 1e12, 10, 1000.0) == pytest.approx(10.0)
