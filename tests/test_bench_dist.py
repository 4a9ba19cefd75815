"""The bench's multi-rank plumbing (replicas only) on CPU: two gloo ranks.

Every rank times its own replica; rank 0 reports the slowest rank's time and the FLOPs of all
ranks. This checks the reductions, the barrier and the rank environment with world size 2.
"""
import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, lr, w = bench.rank_env()
        bench.barrier()
        ms, flops = bench.aggregate(local_ms=1.0 + 2.0 * rank, local_flops=10.0 * (rank + 1))
        out.put((r, lr, w, ms, flops, bench.reduce_max(-rank), bench.reduce_sum(0.5)))
        bench.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[:3] for r in results] == [(0, 0, 2), (1, 1, 2)]
    for _, _, _, ms, flops, mx, sm in results:
        assert ms == pytest.approx(3.0)          # slowest rank
        assert flops == pytest.approx(30.0)      # all ranks' work
        assert mx == pytest.approx(0.0)
        assert sm == pytest.approx(1.0)


def test_single_process_is_identity():
    import bench
    assert bench.aggregate(2.5, 7.0) == (2.5, 7.0)
    assert bench.reduce_max(3.0) == 3.0
