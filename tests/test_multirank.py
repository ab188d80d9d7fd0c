"""The N > 1 host logic of bench.py on world-size-2 gloo ranks (CPU only).

Each rank joins the process group the way bench.py does under torchrun, then
checks the pieces the whole-job number rests on: every rank takes the same
collective steps, the timing is the max over ranks, and the aggregate counts
every rank's work over the slowest rank's time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup(world, backend="gloo")
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(world)
    ms_local = 10.0 + 5.0 * rank          # rank 1 is the slow one
    ms_max = bench.max_over_ranks(ms_local, world)
    tops = bench.aggregate_tops(1000, world, 2.0 * 16 * 4096 * 4096, ms_max)
    bench.barrier(world)
    dist.destroy_process_group()
    out.put((rank, ms_max, tops))


def test_two_gloo_ranks_max_timing_and_weak_aggregate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    assert codes == [0, 0], codes
    res = sorted(q.get(timeout=5) for _ in range(world))
    ops = 2.0 * 16 * 4096 * 4096
    for rank, ms_max, tops in res:
        assert ms_max == 15.0                       # the slowest rank's time on every rank
        assert tops == pytest.approx(1000 * 2 * ops / 15e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate_tops(10, 1, 1e12, 1000.0) == pytest.approx(10.0)   # 1e13 ops in 1 s
