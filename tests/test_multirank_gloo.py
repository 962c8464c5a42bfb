"""Multi-process host logic of the benchmark on CPU (gloo, world size 2).

The path partitions into independent (layer, sequence, KV head) units, so
N GPUs run N independent replicas with no collective in the data path; the
only cross-rank steps are the barrier and the max-over-ranks step time.
These tests run two gloo ranks on the CPU and check that reduction, the
replica seeding (different data per rank) and the whole-job aggregate.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import datagen as DG
        local_ms = 1.5 + rank  # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, dist, "cpu")
        lay = DG.workload2_layer(bench.replica_layer_offset(rank), "cpu", N=64)
        checksum = float(lay.k.float().sum())
        dist.barrier()
        value = bench.whole_job_value(1000.0, world, ms)
        out_q.put((rank, ms, checksum, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_replicas():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    # both ranks see the slowest rank's time
    assert res[0][1] == res[1][1] == pytest.approx(2.5)
    # replicas hold different data
    assert res[0][2] != res[1][2]
    # whole-job value = all ranks' work / max time
    assert res[0][3] == pytest.approx(1000.0 * 2 / 2.5e-3)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, None, "cpu") == 3.25
    assert bench.replica_layer_offset(0) == 0
