"""The benchmark's cross-rank steps on CPU (no GPU): rank and world size from the
launcher's environment, the max-over-ranks time, the agreement of all ranks on parity
(so that every rank stops together), and the whole-job rate, with two `gloo` processes
and in one process."""
import os
import queue
import socket
from datetime import timedelta

import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, w, lr = bench.rank_info()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(1.5 + rank, dist, "cpu")       # rank 1 is the slower one
        ok_all = bench.all_ranks_ok(True, dist, "cpu")
        ok_one = bench.all_ranks_ok(rank == 0, dist, "cpu")      # one rank fails: all stop
        rate = bench.whole_job_rate(1000.0, w, ms)
        out.put((rank, r, w, lr, ms, ok_all, ok_one, rate))
    finally:
        dist.destroy_process_group()


def test_cross_rank_steps_world_size_2():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted(out.get(timeout=120) for _ in range(2))
    except queue.Empty:
        got = []
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    assert len(got) == 2
    for rank, r, w, lr, ms, ok_all, ok_one, rate in got:
        assert (r, w, lr) == (rank, 2, rank)
        assert ms == 2.5                      # the slowest rank's time on every rank
        assert ok_all is True and ok_one is False
        assert rate == 1000.0 * 2 / 2.5e-3    # units of both ranks over the max time


def test_cross_rank_steps_single_process():
    assert bench.max_over_ranks(3.0) == 3.0
    assert bench.all_ranks_ok(False) is False and bench.all_ranks_ok(True) is True
    assert bench.whole_job_rate(10.0, 1, 1000.0) == 10.0
