"""The multi-rank host path of bench.py on CPU: two gloo ranks.

bench.py runs one replica of the workload per rank (weak scaling, no collective on
the data path) and reports all ranks' steps over the slowest rank's time.  These
tests run that reduction and the replica seeding with world size 2 over gloo.
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import bench
    from block_diffusion_attention_prefix_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [120.0, 80.0][rank]
        t_max = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        value = bench.weak_scaling_value(world, 1000, t_max)
        seed = bench.replica_seed(7, rank)
        w = W.get("tiny_f32")
        k, _ = W.prefix_kv(w, seed)
        digest = float(k.double().sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, (t_max, value, seed, digest))
        q.put((rank, gathered))
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_reduction():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        g = results[rank]
        assert g[0][0] == g[1][0] == 120.0                     # every rank sees the slowest time
        assert g[0][1] == pytest.approx(2 * 1000 / 0.120)      # all ranks' steps / slowest time
        assert (g[0][2], g[1][2]) == (7, 8)                   # replica seeds differ per rank
        assert g[0][3] != g[1][3]                             # so the replicas' inputs differ


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(42.0, 1, torch.device("cpu")) == 42.0
    assert bench.weak_scaling_value(1, 100, 50.0) == pytest.approx(2000.0)
