"""The benchmark's multi-rank plumbing (barrier, max over ranks, whole-job aggregation)
with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.dist_env() == (rank, rank, world)
        bench.barrier(world)
        step_s = 0.5 + 0.25 * rank                     # the slower rank decides
        m = bench.max_over_ranks(step_s, world)
        v = bench.aggregate(100e12, world, m, 1)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, m, v in res:
        assert m == pytest.approx(0.75)
        assert v == pytest.approx(2 * 100.0 / 0.75)   # 2 ranks x 100 TFLOP over 0.75 s


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(1.25, 1) == 1.25
    assert bench.aggregate(50e12, 1, 0.5, 1) == pytest.approx(100.0)
