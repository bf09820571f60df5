"""The N > 1 benchmark path on CPU: independent replicas, one per rank, timed
by the slowest rank (world size 2, gloo backend, no GPU).

Every (batch element, KV head) unit of the method is independent, so ranks
run replicas with no collective on the data path; torch.distributed is only
used for the barrier and the max-over-ranks time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 20.0][rank]  # rank 1 is the slow one
        ms_max = bench.max_over_ranks(local_ms, world)
        dist.barrier()
        q.put((rank, ms_max, bench.replica_throughput(world, 8, 100, ms_max)))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_report_the_slowest_rank():
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
    for rank, ms_max, tput in res:
        assert ms_max == 20.0                      # max over ranks, seen by every rank
        assert tput == pytest.approx(2 * 8 * 100 / 0.020)  # both replicas' tokens / slowest time


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.replica_throughput(1, 8, 10, 2.0) == pytest.approx(40000.0)
