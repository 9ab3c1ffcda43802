"""Host logic of the multi-rank benchmark on CPU with gloo, world size 2.

Every rank processes its own batch (weak scaling); the reported time is the
max over ranks and the value counts the units of all ranks."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench.dist_init("gloo")
    assert (w, r) == (world, rank)
    local_seconds = 1.0 + rank          # rank 1 is the slow one
    tmax = bench.max_over_ranks(local_seconds)
    value = bench.weak_scaling_value(100.0, steps=4, world=w, max_seconds=tmax)
    bench.barrier()
    # each rank draws its own activation batch
    import workloads
    x = workloads.llama_acts(0, 2, stream=rank)
    q.put((rank, tmax, value, float(x.astype("float64").sum())))
    torch.distributed.destroy_process_group()


def test_weak_scaling_aggregation_two_ranks():
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
    (r0, t0, v0, s0), (r1, t1, v1, s1) = out
    assert t0 == t1 == 2.0                 # max over ranks
    assert v0 == v1 == 100.0 * 4 * 2 / 2.0  # all ranks' units / slowest time
    assert s0 != s1                        # different batches per rank


def test_single_process_is_world_one(monkeypatch):
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_info() == (1, 0, 0)
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.weak_scaling_value(10.0, 2, 1, 4.0) == 5.0
