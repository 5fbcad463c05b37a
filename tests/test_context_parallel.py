"""The context-parallel split of the prefix on CPU: key ranges, the exchange, the
merge order and the replicated cache, with two gloo ranks.

The compute steps (partial over a range, merge of the partials, in-block part)
run through the CPU oracle here, so these tests check the host-side flow of
ContextParallelLayer -- that the ranks' ranges partition the prefix, that the one
all-gather delivers every rank's partial in range order, that the merge leaves
reusing heads' cache rows alone, and that every rank ends with the same cache and
output -- against the oracle's single-process result over the whole prefix.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_diffusion_attention_prefix_b200.context_parallel import shard_range


@pytest.mark.parametrize("n", [0, 1, 63, 64, 65, 1000, 100_000, 800_000])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_ranges_partition_the_prefix(n, world):
    ranges = [shard_range(n, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == n
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0, "ranges must be contiguous and in rank order"
    for r, (n0, n1) in enumerate(ranges):
        assert 0 <= n0 <= n1 <= n
        if r < world - 1:
            assert n0 % 64 == 0 and n1 % 64 == 0 or n1 == n


class OracleOps:
    """The three compute steps of a context-parallel step on the CPU oracle (float64)."""

    def __init__(self, scale):
        self.scale = scale

    def _reuse(self, g, hq):
        from oracle import flashblock as OF
        sim = None if g.head_sim is None else g.head_sim.numpy()
        return OF.decisions(g.mask.numpy(), g.first_step, g.tau, sim, g.gamma, hq)

    def partial(self, shape, q, k, v, g, a, l, ws):
        from oracle import flashblock as OF
        _, reuse = self._reuse(g, q.shape[1])
        A, L = OF.prefix_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), self.scale)
        rec = torch.from_numpy(~reuse)
        a[rec] = torch.from_numpy(A)[rec].float()
        l[rec] = torch.from_numpy(L)[rec].float()

    def merge(self, shape, a_parts, a_stride, l_parts, l_stride, n, g, a_out, l_out):
        from oracle import attention as OA
        b, hq, B, D = a_out.shape
        rows = b * hq * B
        parts = [(a_parts[p].reshape(b, hq, B, D).double().numpy(), l_parts[p][:rows].reshape(b, hq, B).double().numpy())
                 for p in range(n)]
        A, L = OA.merge_all(parts)
        _, reuse = self._reuse(g, hq)
        rec = torch.from_numpy(~reuse)
        a_out[rec] = torch.from_numpy(A)[rec].float()
        l_out[rec] = torch.from_numpy(L)[rec].float()

    def block_merge(self, shape, q, kb, vb, g, a_out, l_out, a_full, l_full, dM, dR, ws):
        from oracle import attention as OA
        from oracle import flashblock as OF
        M, reuse = self._reuse(g, q.shape[1])
        Ai, Li = OF.block_attention(q.double().numpy(), kb.double().numpy(), vb.double().numpy(), self.scale)
        A, L = OA.merge(a_out.double().numpy(), l_out.double().numpy(), Ai, Li)
        a_full.copy_(torch.from_numpy(A))
        l_full.copy_(torch.from_numpy(L))
        dM.copy_(torch.from_numpy(M))
        dR.copy_(torch.from_numpy(reuse.astype(np.uint8)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs():
    from block_diffusion_attention_prefix_b200 import workloads as W
    w = W.get("tiny_f32").with_(h_q=4, h_kv=2, n_prefix=300, steps=6)
    k, v = W.prefix_kv(w, 5)
    return w, k, v, list(W.block_schedule(w, 5))


def _worker(rank, world, port, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    from block_diffusion_attention_prefix_b200.context_parallel import ContextParallelLayer
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, k, v, sched = _inputs()
        n0, n1 = shard_range(w.n_prefix, world, rank)
        layer = ContextParallelLayer(None, w.batch, w.h_q, w.h_kv, w.head_dim, w.block, w.n_prefix,
                                     k[:, :, n0:n1].contiguous(), v[:, :, n0:n1].contiguous(), rank, world,
                                     ops=OracleOps(1 / math.sqrt(w.head_dim)))
        out = []
        for s in sched:
            layer.step(s.q, s.k_blk, s.v_blk, s.mask, s.first, w.tau)
            out.append(tuple(t.numpy().copy() for t in (layer.a_full, layer.l_full, layer.a_out, layer.l_out,
                                                         layer.dec_M, layer.dec_reuse)))
        q_out.put((rank, (n0, n1), out))
    finally:
        dist.destroy_process_group()


def test_two_rank_context_parallel_step_equals_whole_prefix():
    from oracle import flashblock as OF
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in procs:
        rank, rng, out = q.get(timeout=180)
        results[rank] = (rng, out)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w, k, v, sched = _inputs()
    assert results[0][0][1] == results[1][0][0] and results[0][0][1] > 0, "both ranks hold keys"
    ref = OF.CachedBlockAttention(k.double().numpy(), v.double().numpy(), w.h_q, 1 / math.sqrt(w.head_dim))
    kinds = set()
    for i, s in enumerate(sched):
        r = ref.step(s.q.double().numpy(), s.k_blk.double().numpy(), s.v_blk.double().numpy(), s.mask.numpy(),
                     s.first, w.tau)
        kinds.add(bool(r.reuse.any()))
        for rank in range(world):
            a_full, l_full, a_out, l_out, dM, dR = results[rank][1][i]
            assert np.array_equal(dM, r.M) and np.array_equal(dR.astype(bool), r.reuse)
            for got, want in ((a_full, r.a_full), (l_full, r.l_full), (a_out, r.a_out), (l_out, r.l_out)):
                assert np.abs(got.astype(np.float64) - want).max() <= 1e-5, f"step {i} rank {rank}"
        for t0, t1 in zip(results[0][1][i], results[1][1][i]):
            assert np.array_equal(t0, t1), "every rank holds the same cache and output"
    assert kinds == {True, False}, "the schedule must mix reuse and recompute steps"
