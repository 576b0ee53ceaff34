"""The benchmark's multi-GPU path on CPU: two gloo ranks run the host logic
bench.py uses under torchrun (max of the timed regions over ranks, sum of the
work units, barriers), and the reference arm does its work on rank 0 only."""
import io
import os
import socket
import contextlib

import pytest
import torch.multiprocessing as tmp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.rank_env() == (rank, rank, world)
        bench.barrier(world)
        ms, units = bench.reduce_over_ranks(10.0 + 5.0 * rank, 100 * (rank + 1), world)
        bench.barrier(world)
        q.put((rank, ms, units))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_max_time_and_sum_units():
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, units in res:
        assert ms == 15.0          # the slower rank's timed region
        assert units == 300.0      # all ranks' work


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_over_ranks(3.5, 7, 1) == (3.5, 7.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3"])
    assert out.getvalue() == ""


def test_reference_arm_line(monkeypatch):
    import json
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3",
                    "--cpu-seconds", "0.5"])
    line = json.loads(out.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["higher_is_better"] is True
