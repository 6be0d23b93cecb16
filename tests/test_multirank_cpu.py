"""The bench's N > 1 path on CPU: two gloo ranks run the same aggregation code the GPU
ranks run (max over ranks of the device time, whole-job throughput over the slowest rank).
Decode has no exchange step, so this is the only cross-rank logic."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [0.25, 0.75][rank]
        slow = bench.slowest_rank_seconds(mine, dist, "cpu")
        gbs = bench.job_throughput(1_000_000_000, 3, world, slow)
        dist.barrier()
        q.put((rank, slow, gbs))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slow, gbs in res:
        assert slow == 0.75
        assert gbs == pytest.approx(2 * 3 * 1.0 / 0.75)


def test_single_rank_is_identity():
    import bench
    assert bench.slowest_rank_seconds(1.5) == 1.5
    assert bench.job_throughput(2_000_000_000, 4, 1, 2.0) == pytest.approx(4.0)
