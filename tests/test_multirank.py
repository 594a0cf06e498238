"""The N > 1 host path of bench.py on CPU: two gloo ranks exercise the
max-over-ranks timing reduction and the whole-job throughput aggregation
(weak scaling, no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        assert bench.dist_env() == (world, rank, rank)
        # rank r "took" 1 + r seconds for 100 steps; the job time is the max
        got = bench.aggregate(100, 1.0 + rank, world, torch.device("cpu"))
        bench.barrier()
        q.put((rank, got["seconds"], got["value"]))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_takes_max_time_and_sums_units():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, seconds, value in res:
        assert seconds == pytest.approx(2.0)            # max over ranks
        assert value == pytest.approx(2 * 100 / 2.0)    # all ranks' units / max time


def test_single_rank_aggregation_is_identity():
    import bench
    got = bench.aggregate(50, 0.5, 1, torch.device("cpu"))
    assert got == {"seconds": 0.5, "value": 100.0}
