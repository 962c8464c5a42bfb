"""Multi-process host logic of the benchmark on CPU (gloo, world size 2).

The path partitions into independent (layer, sequence, KV head) units, so N
GPUs either split the KV heads (and, past the head count, the layers) of one
workload -- the default -- or run N independent replicas; neither has a
collective in the data path, the only cross-rank steps being the barrier and
the max-over-ranks step time.  These tests run gloo ranks on the CPU and
check that reduction, the replica seeding (different data per rank), the
whole-job aggregate, that the head partition covers every unit exactly once
in equal shares, and that the per-rank head slices of a small workload,
computed with the oracle and gathered back, equal the unsharded result.
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


# --------------------------------------------------------------------------- KV-head sharding
def test_shard_plan_covers_every_unit_once():
    import bench
    for world in (1, 2, 3, 4, 6, 8, 12, 16):
        seen = {}
        for r in range(world):
            p = bench.shard_plan(r, world)
            assert p["g1"] > p["g0"] and p["l1"] > p["l0"]
            for l in range(p["l0"], p["l1"]):
                for g in range(p["g0"], p["g1"]):
                    assert (l, g) not in seen, (world, l, g)
                    seen[(l, g)] = r
        assert len(seen) == bench.LAYERS * bench.HKV, world
        # equal shares (the whole-job value counts the workload once)
        sizes = {(bench.shard_plan(r, world)["l1"] - bench.shard_plan(r, world)["l0"]) *
                 (bench.shard_plan(r, world)["g1"] - bench.shard_plan(r, world)["g0"]) for r in range(world)}
        if bench.LAYERS % (world // __import__("math").gcd(world, bench.HKV)) == 0:
            assert len(sizes) == 1, (world, sizes)


def _shard_worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import math

        import bench
        import datagen as DG
        import oracle as O
        layers, hkv, G, Nt = 3, 4, 8, 96
        plan = bench.shard_plan(rank, world, layers=layers, hkv=hkv)
        parts = []
        for l in range(plan["l0"], plan["l1"]):
            lay = DG.workload2_layer(l, "cpu", N=Nt)
            q, k, v = bench.shard_layer(lay.q, lay.k, lay.v, plan, G)
            out = torch.empty((1, q.shape[1], 128), dtype=torch.float64)
            for g in range(k.shape[1]):
                res = O.decode_unit(q[0, g * G:(g + 1) * G].float().numpy(), k[0, g].float().numpy(),
                                    v[0, g].float().numpy(), Nt, rule="envelope", page_size=16,
                                    budget={"kind": "topk", "k": 2}, scale=1 / math.sqrt(128))
                out[0, g * G:(g + 1) * G] = torch.from_numpy(res.out)
            parts.append(out)
        mine = torch.cat(parts)
        gathered = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(gathered, mine)  # test-side reassembly only: the benchmark has no collective
        plans = [bench.shard_plan(r, world, layers=layers, hkv=hkv) for r in range(world)]
        full = bench.reassemble_heads(gathered, plans, G, layers=layers)
        out_q.put((rank, full.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_rank_head_sharding_reassembles_the_whole_workload():
    """Two gloo ranks each compute (with the oracle) the decode of their KV
    heads' shard of a small 3-layer workload; gathering the head slices back
    gives exactly the unsharded computation."""
    import math

    import numpy as np

    import datagen as DG
    import oracle as O
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    layers, G, Nt = 3, 8, 96
    ref = np.empty((layers, 32, 128))
    for l in range(layers):
        lay = DG.workload2_layer(l, "cpu", N=Nt)
        for g in range(4):
            r = O.decode_unit(lay.q[0, g * G:(g + 1) * G].float().numpy(), lay.k[0, g].float().numpy(),
                              lay.v[0, g].float().numpy(), Nt, rule="envelope", page_size=16,
                              budget={"kind": "topk", "k": 2}, scale=1 / math.sqrt(128))
            ref[l, g * G:(g + 1) * G] = r.out
    for _, full in res:
        assert np.array_equal(full, ref)
