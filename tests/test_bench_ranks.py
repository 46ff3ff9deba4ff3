"""The bench's multi-rank host logic on CPU: two `gloo` ranks (world size 2).

- Timings reduce to the element-wise maximum over ranks on every rank.
- The whole-job rate is the work of all ranks over the slowest rank's time.
- The reference arm runs on rank 0 only: the other ranks return at once and
  print nothing.
"""
import contextlib
import io
import os
import socket
import sys
import types

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank timings: rank r is slowest on entry r
        mine = [1.0 + (rank == 0), 5.0 + 3 * (rank == 1), 0.25]
        got = bench.max_over_ranks(mine, world, "cpu")
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            if rank != 0:
                args = types.SimpleNamespace(steps=1, warmup=0)
                bench.run_reference(args, rank, world)
        out[rank] = (got, buf.getvalue())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank in range(world):
        got, printed = res[rank]
        assert got == [2.0, 8.0, 0.25]
        assert printed == ""


def test_single_rank_is_a_no_op_and_rate_is_aggregate():
    import bench
    assert bench.max_over_ranks([3.0, 1.0], 1, "cpu") == [3.0, 1.0]
    assert bench.aggregate_rate(10.0, 4, 2.0) == pytest.approx(20.0)
