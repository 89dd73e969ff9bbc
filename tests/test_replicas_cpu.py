"""The benchmark's multi-GPU path on the CPU: two gloo ranks running independent replicas.

The layer does not shard, so N GPUs run N replicas with no data-path collective; the only
collectives are a barrier and the maximum of the per-rank step times.  This runs that plumbing with
world size 2 on the CPU: rendezvous, barrier, max over ranks, and the whole-job throughput formula.
"""
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
    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_setup(world)
    bench.barrier(w)
    ms = [3.0, 5.0][r]                       # rank 1 is the slow one
    slowest = bench.max_over_ranks(ms, w)
    T = 4096
    q.put((r, w, local, slowest, w * T / (slowest * 1e-3)))
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_replicas_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[0] for o in out] == [0, 1]
    for r, w, local, slowest, value in out:
        assert w == 2 and local == r
        assert slowest == pytest.approx(5.0)                 # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 4096 / 5e-3)       # tokens of all replicas / slowest time
