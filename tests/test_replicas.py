"""The N > 1 path of bench.py on CPU: world-size-2 gloo ranks.

The GEMV path shards into independent replicas (one per GPU, no data-path
collective), so what runs across ranks is host logic: the barrier around the
timed region, the max over ranks of each timing, the whole-job throughput
(bytes of every replica over the slowest rank's time), and the reference arm
running on rank 0 only.  These tests run that logic with the gloo backend."""
import os
import socket
from datetime import timedelta

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        steps = 100
        local_ms = 10.0 + 5.0 * rank                      # rank 1 is the slower replica
        bench.barrier(world)
        ms = bench.allreduce_max(local_ms, world)
        bench.barrier(world)
        value = bench.replica_value(bench.STEP_BYTES, world, ms / steps)
        ref = bench.run_reference(None, world, rank, rank) if rank != 0 else "rank0"
        q.put((rank, ms, value, ref))
    finally:
        dist.destroy_process_group()


def _run(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    codes = [p.exitcode for p in procs]
    assert codes == [0] * world, codes
    return sorted(q.get(timeout=10) for _ in range(world))


def test_two_replicas_take_the_slowest_rank_and_sum_the_bytes():
    res = _run(2)
    slowest = 15.0
    for rank, ms, value, ref in res:
        assert ms == slowest                                  # every rank sees the max
        assert value == pytest.approx(2 * bench.STEP_BYTES / (slowest / 100 * 1e-3) / 1e9)
    assert res[1][3] is None                                  # the reference arm runs on rank 0 only


def test_replica_value_is_weak_scaling():
    one = bench.replica_value(bench.STEP_BYTES, 1, 1.5)
    assert bench.replica_value(bench.STEP_BYTES, 4, 1.5) == pytest.approx(4 * one)
    assert bench.replica_value(bench.STEP_BYTES, 4, 3.0) == pytest.approx(2 * one)
