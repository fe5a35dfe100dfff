"""Host logic of the multi-GPU bench path on CPU: two `gloo` ranks.

The decode path shards by replica (every rank runs the whole chain on its own
batch), so the only cross-rank steps are the timing barrier and the
max-over-ranks reduction of the step time; both are exercised here.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q) -> None:
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    import torch.distributed as dist
    try:
        assert bench.dist_init("gloo") == world
        ms = 2.0 + 3.0 * rank          # rank 1 is the slow one
        bench.barrier()
        ms_max = bench.reduce_max(ms)
        q.put((rank, ms_max, bench.whole_job_throughput(world, 4, ms_max)))
        bench.barrier()
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_rank_timing_reduction():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms_max, thr in got:
        assert ms_max == pytest.approx(5.0)            # max over ranks, seen by every rank
        assert thr == pytest.approx(2 * 4 / 5.0e-3)     # all ranks' tokens over the slowest rank's time


def test_single_process_is_identity():
    import bench
    assert bench.reduce_max(3.5) == 3.5
    assert bench.whole_job_throughput(1, 8, 2.0) == pytest.approx(4000.0)
