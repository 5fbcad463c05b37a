"""GPU parity of the context-parallel split of the prefix, its ranks emulated on one GPU.

Each emulated rank holds its own contiguous key range of the prefix (a copy, as a
rank's shard would be), computes its partial with fb_prefix_attn, the partials
are stacked as an all-gather would leave them, fb_merge_partials merges them in
range order into the cache and fb_block_merge finishes the step.  At every step of
a seeded schedule the decisions must match the oracle's over the whole prefix bit
for bit and the cache and outputs must be within the parity tolerance; a single
range must give its partial back bit for bit.
"""
import math

import numpy as np
import pytest
import torch

from block_diffusion_attention_prefix_b200 import workloads as W
from block_diffusion_attention_prefix_b200.context_parallel import ContextParallelLayer, shard_range
from oracle import flashblock as OF

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}


def f64(t):
    return t.detach().to("cpu").double().numpy()


def close(got, want, tol, what):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(want)), f"{what}: -inf pattern differs"
    both = np.isneginf(got) & np.isneginf(want)
    err = np.abs(np.where(both, 0.0, got) - np.where(both, 0.0, want)).max()
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


def ws_for(fb, shape):
    n = fb.fb_workspace_bytes(shape)
    return torch.zeros(((n + 15) // 16 * 16,), device="cuda", dtype=torch.uint8)


@pytest.mark.parametrize("name,n_prefix,P,gamma", [
    ("dlm8b_b4", 5000, 1, None),
    ("dlm8b_b4", 5000, 2, None),
    ("dlm8b_b4", 5000, 3, None),
    ("dlm8b_b4", 130, 5, None),       # more ranges than key tiles: empty ranges merge as (0, -inf)
    ("dlm8b_b16", 4097, 4, None),     # 64 rows per KV head: the tcgen05 pass on every range
    ("tiny_f32", 1000, 3, None),
    ("video", 3000, 3, 0.95),         # per-head gate: only recomputing heads' cache rows change
])
def test_ranges_merged_equal_whole_prefix(fb, name, n_prefix, P, gamma):
    w = W.get(name).with_(n_prefix=n_prefix, steps=5)
    if name == "video":
        w = w.with_(block=16, h_q=6, h_kv=6, tau=17)
    seed = 21
    k, v = W.prefix_kv(w, seed)
    sched = list(W.block_schedule(w, seed))
    dt = w.dtype
    full = fb.make_shape(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, w.n_prefix, dt)
    ranges = [shard_range(w.n_prefix, P, p) for p in range(P)]
    shards = [(k[:, :, n0:n1].contiguous().cuda(), v[:, :, n0:n1].contiguous().cuda()) for n0, n1 in ranges]
    sshapes = [fb.make_shape(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, n1 - n0, dt) for n0, n1 in ranges]
    sws = [ws_for(fb, s) for s in sshapes]
    b, hq, B, D = w.batch, w.h_q, w.block, w.head_dim
    a_parts = torch.zeros((P, b, hq, B, D), device="cuda")
    l_parts = torch.zeros((P, b, hq, B), device="cuda")
    a_out = torch.zeros((b, hq, B, D), device="cuda")
    l_out = torch.full((b, hq, B), float("-inf"), device="cuda")
    a_full = torch.zeros((b, hq, B, D), device="cuda", dtype=w.torch_dtype)
    l_full = torch.zeros((b, hq, B), device="cuda")
    dM = torch.zeros((b,), device="cuda", dtype=torch.int32)
    dR = torch.zeros((b, hq), device="cuda", dtype=torch.uint8)
    ws = ws_for(fb, full)
    ref = OF.CachedBlockAttention(f64(k), f64(v), hq, 1 / math.sqrt(D))
    kinds = set()
    for s in sched:
        sim = None if s.sim is None else s.sim.cuda()
        gate = fb.make_gate(s.mask.cuda(), s.first, w.tau, sim, gamma or 0.0)
        q = s.q.cuda()
        for p in range(P):
            fb.fb_prefix_attn(sshapes[p], q, shards[p][0], shards[p][1], gate, a_parts[p], l_parts[p], sws[p])
        prev_a, prev_l = a_out.clone(), l_out.clone()
        fb.fb_merge_partials(full, a_parts, b * hq * B * D, l_parts, b * hq * B, P, gate, a_out, l_out)
        fb.fb_block_merge(full, q, s.k_blk.cuda(), s.v_blk.cuda(), gate, a_out, l_out, a_full, l_full, dM, dR, ws)
        torch.cuda.synchronize()
        r = ref.step(f64(s.q), f64(s.k_blk), f64(s.v_blk), s.mask.numpy(), s.first, w.tau,
                     None if s.sim is None else s.sim.numpy(), gamma or 0.0)
        kinds.add((bool(r.reuse.any()), bool((~r.reuse).any())))
        tag = f"{name} P={P} step {s.index}"
        assert np.array_equal(dM.cpu().numpy(), r.M), f"{tag}: M"
        assert np.array_equal(dR.cpu().numpy().astype(bool), r.reuse), f"{tag}: reuse"
        tol = TOL[dt]
        close(f64(a_out), r.a_out, tol, f"{tag} A_out")
        close(f64(l_out), r.l_out, tol, f"{tag} L_out")
        close(f64(a_full), r.a_full, tol, f"{tag} A_full")
        close(f64(l_full), r.l_full, tol, f"{tag} L_full")
        for bi in range(b):
            for h in range(hq):
                if r.reuse[bi, h]:   # reusing heads' cache rows untouched bit for bit
                    assert torch.equal(a_out[bi, h], prev_a[bi, h]) and torch.equal(l_out[bi, h], prev_l[bi, h])
                elif P == 1:         # one range: the merge gives the partial back bit for bit
                    assert torch.equal(a_out[bi, h], a_parts[0, bi, h]) and torch.equal(l_out[bi, h], l_parts[0, bi, h])
    assert fb.fb_device_error() == 0
    assert any(x for x, _ in kinds), "want reuse decisions in the schedule"


def test_layer_single_rank_through_libfb(fb):
    # ContextParallelLayer with one rank (no process group): the libfb ops end to end
    w = W.get("dlm8b_b4").with_(n_prefix=3000, steps=4)
    k, v = W.prefix_kv(w, 8)
    layer = ContextParallelLayer(fb, w.batch, w.h_q, w.h_kv, w.head_dim, w.block, w.n_prefix, k.cuda(), v.cuda(),
                                 0, 1)
    ref = OF.CachedBlockAttention(f64(k), f64(v), w.h_q, 1 / math.sqrt(w.head_dim))
    for s in W.block_schedule(w, 8):
        layer.step(s.q.cuda(), s.k_blk.cuda(), s.v_blk.cuda(), s.mask.cuda(), s.first, w.tau)
        torch.cuda.synchronize()
        r = ref.step(f64(s.q), f64(s.k_blk), f64(s.v_blk), s.mask.numpy(), s.first, w.tau)
        assert np.array_equal(layer.dec_reuse.cpu().numpy().astype(bool), r.reuse)
        close(f64(layer.a_full), r.a_full, 2e-2, f"step {s.index} A_full")
        close(f64(layer.a_out), r.a_out, 2e-2, f"step {s.index} A_out")
    assert fb.fb_device_error() == 0
