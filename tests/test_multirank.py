"""Host logic of multi-GPU runs, on CPU with the gloo backend (world size 2).

Every rank verifies its own independent sequences (weak scaling, no collective
on the data path); the benchmark only reduces timings: the whole-job time is
the maximum over ranks and the units are summed.
"""
import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench.dist_env()
        ms, units, value = bench.aggregate(10.0 + 5.0 * rank, 100.0 + rank, ws, device="cpu")
        bench.barrier(ws)
        ref = bench.run_reference(bench_args(), ws, r) if r != 0 else "skipped"
        queue.put((rank, ws, local, ms, units, value, ref))
    finally:
        dist.destroy_process_group()


def bench_args():
    import argparse
    return argparse.Namespace(steps=1, warmup=3, batch=1, budget=22, layers=48, seed=2, state_dtype="f32")


@pytest.mark.timeout(180)
def test_two_rank_aggregation_gloo():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=150) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ws, local, ms, units, value, ref in results:
        assert ws == 2 and local == rank
        assert ms == pytest.approx(15.0)           # max over ranks
        assert units == pytest.approx(201.0)       # sum over ranks
        assert value == pytest.approx(201.0 / 0.015)
    # the reference arm runs on rank 0 only; other ranks print nothing
    assert results[1][6] is None


def test_single_rank_aggregation_is_local():
    import bench
    ms, units, value = bench.aggregate(20.0, 50.0, 1)
    assert (ms, units) == (20.0, 50.0) and value == pytest.approx(2500.0)
