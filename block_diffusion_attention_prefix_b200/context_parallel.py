"""Context-parallel split of the prefix over ranks (one GPU per rank).

FlashBlock technical summary (gist.science 2602.05305), "2. Methodology / Core
mechanism": the log-space merge equation combines partial attention results over
disjoint key sets into the result over their union.  So the out-of-block set
J_out -- the prefix, whose K/V read is the whole cost of a recompute step -- can
be cut into P contiguous key ranges, one per rank:

  1. every rank computes, for the rows whose gate says recompute, the partial
     (A, L) over its own range of the prefix (fb_prefix_attn on its K/V shard);
  2. one all-gather moves the P partials (b * H_q * B * (D + 1) fp32 per rank)
     to every rank -- the only exchange of the step;
  3. every rank merges them in range order (fb_merge_partials) into its replica
     of the cache (A_out, L_out), so all replicas hold the same bits;
  4. every rank runs the in-block part and the final merge (fb_block_merge).

Reuse steps change no cache row (the gathered partials of reusing heads are
ignored by the merge), so the replicas stay equal without further traffic.  The
gate is evaluated on the device from the step's mask on every rank, so the host
does not know which steps reuse and every rank runs the same collective every
step.  The compute steps go through an `ops` object (libfb by default); the
host-side flow -- ranges, gather, merge order -- is the same whatever computes.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

__all__ = ["shard_range", "GateSpec", "LibfbOps", "ContextParallelLayer"]


def shard_range(n_prefix: int, world: int, rank: int, align: int = 64):
    """Contiguous key range [n0, n1) of `rank`: near-equal shares in whole multiples
    of `align` keys (the passes' key tile), the last rank taking what is left.  The
    ranges of ranks 0 .. world-1 are disjoint, in order, and cover [0, n_prefix)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    per = -(-n_prefix // (world * align)) * align
    n0 = min(n_prefix, rank * per)
    n1 = n_prefix if rank == world - 1 else min(n_prefix, n0 + per)
    return n0, n1


@dataclasses.dataclass
class GateSpec:
    """The gate of one step as given by the caller (device mask, optional head similarity)."""
    mask: torch.Tensor
    first_step: bool
    tau: int
    head_sim: Optional[torch.Tensor] = None
    gamma: float = 0.0


class LibfbOps:
    """The compute steps of a context-parallel step, through libfb (device tensors)."""

    def __init__(self, fb):
        self.fb = fb

    def _gate(self, g: GateSpec):
        return self.fb.make_gate(g.mask, g.first_step, g.tau, g.head_sim, g.gamma)

    def workspace(self, shape):
        n = self.fb.fb_workspace_bytes(shape)
        return torch.zeros(((n + 15) // 16 * 16,), device="cuda", dtype=torch.uint8)

    def partial(self, shape, q, k, v, gate: GateSpec, a, l, ws):
        self.fb.fb_prefix_attn(shape, q, k, v, self._gate(gate), a, l, ws)

    def merge(self, shape, a_parts, a_stride, l_parts, l_stride, n_parts, gate: GateSpec, a_out, l_out):
        self.fb.fb_merge_partials(shape, a_parts, a_stride, l_parts, l_stride, n_parts, self._gate(gate), a_out, l_out)

    def block_merge(self, shape, q, k_blk, v_blk, gate: GateSpec, a_out, l_out, a_full, l_full, dec_M, dec_reuse, ws):
        self.fb.fb_block_merge(shape, q, k_blk, v_blk, self._gate(gate), a_out, l_out, a_full, l_full, dec_M,
                               dec_reuse, ws)


class ContextParallelLayer:
    """One attention layer whose prefix is split over the ranks of `group`.

    k_shard / v_shard: this rank's keys and values [b, H_kv, n1 - n0, D] of the
    range shard_range(n_prefix, world, rank).  Holds the replicated cache, the
    outputs and the exchange buffers."""

    def __init__(self, fb, batch, h_q, h_kv, head_dim, block, n_prefix, k_shard, v_shard, rank, world,
                 group=None, ops=None, dtype=None):
        self.fb, self.rank, self.world, self.group = fb, rank, world, group
        self.ops = ops if ops is not None else LibfbOps(fb)
        dev = k_shard.device
        dtype = k_shard.dtype if dtype is None else dtype
        self.n0, self.n1 = shard_range(n_prefix, world, rank)
        if k_shard.shape[2] != self.n1 - self.n0:
            raise ValueError(f"rank {rank} holds keys [{self.n0}, {self.n1}): shard has {k_shard.shape[2]}")
        dt = "f32" if dtype == torch.float32 else "bf16"
        self.shape = fb.make_shape(batch, h_q, h_kv, head_dim, block, n_prefix, dt) if fb else None
        self.shard_shape = fb.make_shape(batch, h_q, h_kv, head_dim, block, self.n1 - self.n0, dt) if fb else None
        self.k, self.v = k_shard, v_shard
        rows = batch * h_q * block
        # one flat buffer per partial: A, then L; padded so every partial's A is 16-byte aligned
        self.a_elems, self.flat = rows * head_dim, -(-rows * (head_dim + 1) // 4) * 4
        f32 = dict(device=dev, dtype=torch.float32)
        # exchange buffers: this rank's partial (A then L, one flat buffer) and all ranks' partials
        self.part = torch.zeros((self.flat,), **f32)
        self.gathered = torch.zeros((world, self.flat), **f32)
        self.a_part = self.part[:self.a_elems].view(batch, h_q, block, head_dim)
        self.l_part = self.part[self.a_elems:self.a_elems + rows].view(batch, h_q, block)
        self.a_out = torch.zeros((batch, h_q, block, head_dim), **f32)
        self.l_out = torch.full((batch, h_q, block), -math.inf, **f32)
        self.a_full = torch.zeros((batch, h_q, block, head_dim), device=dev, dtype=dtype)
        self.l_full = torch.zeros((batch, h_q, block), **f32)
        self.dec_M = torch.zeros((batch,), device=dev, dtype=torch.int32)
        self.dec_reuse = torch.zeros((batch, h_q), device=dev, dtype=torch.uint8)
        self.ws = self.ops.workspace(self.shape) if hasattr(self.ops, "workspace") else None
        self.shard_ws = self.ops.workspace(self.shard_shape) if hasattr(self.ops, "workspace") else None

    def step(self, q, k_blk, v_blk, mask, first_step, tau, head_sim=None, gamma=0.0):
        g = GateSpec(mask, bool(first_step), int(tau), head_sim, float(gamma))
        # 1. this rank's range: partial (A, L) of the recomputing rows
        self.ops.partial(self.shard_shape, q, self.k, self.v, g, self.a_part, self.l_part, self.shard_ws)
        # 2. the one exchange: every rank's partial, in rank (= range) order
        if self.world > 1:
            torch.distributed.all_gather(list(self.gathered.unbind(0)), self.part, group=self.group)
        else:
            self.gathered[0].copy_(self.part)
        # 3. the cache rows of recomputing heads = merge of the partials in range order
        self.ops.merge(self.shape, self.gathered[:, :self.a_elems], self.flat, self.gathered[:, self.a_elems:],
                       self.flat, self.world, g, self.a_out, self.l_out)
        # 4. in-block part and the final merge, on every rank
        self.ops.block_merge(self.shape, q, k_blk, v_blk, g, self.a_out, self.l_out, self.a_full, self.l_full,
                             self.dec_M, self.dec_reuse, self.ws)
        return self.a_full
