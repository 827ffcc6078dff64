"""Multi-process (world size 2, gloo on CPU) check of the replica aggregation
used by bench.py for N GPUs: units add up over ranks, time is the slowest rank."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    from layer_wise_mixed_kvq_b200 import replicas
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert replicas.world() == (rank, world, rank)
        units = 100.0 * (rank + 1)          # ranks did different amounts of work
        ms = 10.0 if rank == 0 else 40.0    # rank 1 is slower
        total, slowest, rate = replicas.aggregate(units, ms)
        replicas.barrier()
        q.put((rank, total, slowest, rate))
    finally:
        dist.destroy_process_group()


def test_aggregate_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, total, slowest, rate in res:
        assert total == 300.0
        assert slowest == 40.0
        assert rate == pytest.approx(300.0 / 0.040)


def test_single_process_is_identity():
    from layer_wise_mixed_kvq_b200 import replicas
    assert replicas.aggregate(5.0, 2.0) == (5.0, 2.0, 2500.0)
