"""GPU parity at the workloads' full sizes, on every row (long context) or on every
row tile (video), against the CPU oracle.

Long context ("Technical summary: FlashBlock", section 4 Results, long-context
scaling from 100k to 800k tokens): the seeded 8-step schedule of each length is
replayed through fb_step -- reuse steps, an M = 0 step and a recompute after
reuses included -- and at every step the decisions must match bit for bit and
A_full, L_full, A_out and L_out of all 128 query rows must be within the bf16
tolerance.  The oracle replays the same schedule one KV-head group at a time
(the gate is per batch element, so every group sees the same decisions), which
keeps its float64 copy of the prefix at one group (2 x 819 MB at 800k) instead
of the whole cache.

Video (section "Adaptive reuse strategies", per-head selection): the 4-step
schedule with the gamma gate at full size (12 heads, 4680 block queries, a
31,200-token prefix); every row of two heads, and in every other head one row
of each of the 37 row tiles of 128 rows the tensor-core pass computes plus the
first and last rows.
"""
import math

import numpy as np
import pytest
import torch

from block_diffusion_attention_prefix_b200 import workloads as W
from oracle import flashblock as OF

pytestmark = pytest.mark.gpu

TOL = 2e-2


def f64(t):
    return t.detach().to("cpu").double().numpy()


def close(got, want, tol, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(want)), f"{what}: -inf pattern differs"
    both = np.isneginf(got) & np.isneginf(want)
    err = np.abs(np.where(both, 0.0, got) - np.where(both, 0.0, want)).max() if got.size else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"
    return err


def gpu_replay(fb, w, k, v, sched):
    """Every step of the schedule through fb_step; the per-step outputs on the host."""
    layer = fb.CachedAttentionLayer(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, k.cuda(), v.cuda())
    out = []
    for s in sched:
        sim = None if s.sim is None else s.sim.cuda()
        layer.step(s.q.cuda(), s.k_blk.cuda(), s.v_blk.cuda(), s.mask.cuda(), s.first, w.tau, sim, w.gamma or 0.0)
        torch.cuda.synchronize()
        out.append(dict(M=layer.dec_M.cpu().numpy(), reuse=layer.dec_reuse.cpu().numpy().astype(bool),
                        a_full=layer.a_full.cpu(), l_full=layer.l_full.cpu(), a_out=layer.a_out.cpu(),
                        l_out=layer.l_out.cpu()))
    assert fb.fb_device_error() == 0
    del layer
    torch.cuda.empty_cache()
    return out


@pytest.mark.parametrize("name,seed", [("long_100k", 5), ("long_200k", 3), ("long_400k", 5), ("long_800k", 3)])
def test_long_context_full_schedule_every_row(fb, name, seed):
    w = W.get(name)
    sched = list(W.block_schedule(w, seed))
    recompute = [s.first or int(s.mask.sum()) >= w.tau for s in sched]
    assert any(recompute[1:]) and not all(recompute), "want reuse steps and a recompute after reuses"
    assert any(int(s.mask.sum()) == 0 for s in sched[1:]), "want an M = 0 step"
    k, v = W.prefix_kv(w, seed)
    got = gpu_replay(fb, w, k, v, sched)

    # reuse steps leave the cache bit for bit untouched (before the oracle runs)
    for prev, cur, rec in zip(got, got[1:], recompute[1:]):
        if not rec:
            assert torch.equal(cur["a_out"], prev["a_out"]) and torch.equal(cur["l_out"], prev["l_out"])

    G, scale = w.group, 1 / math.sqrt(w.head_dim)
    for g in range(w.h_kv):
        hs = slice(g * G, (g + 1) * G)
        ref = OF.CachedBlockAttention(k[:, g:g + 1].double().numpy(), v[:, g:g + 1].double().numpy(), G, scale)
        for s, o in zip(sched, got):
            r = ref.step(f64(s.q[:, hs]), f64(s.k_blk[:, g:g + 1]), f64(s.v_blk[:, g:g + 1]), s.mask.numpy(),
                         s.first, w.tau)
            tag = f"{name} step {s.index} KV group {g}"
            assert np.array_equal(o["M"], r.M), f"{tag}: M"
            assert np.array_equal(o["reuse"][:, hs], r.reuse), f"{tag}: reuse"
            close(f64(o["a_full"][:, hs]), r.a_full, TOL, f"{tag} A_full")
            close(f64(o["l_full"][:, hs]), r.l_full, TOL, f"{tag} L_full")
            close(f64(o["a_out"][:, hs]), r.a_out, TOL, f"{tag} A_out")
            close(f64(o["l_out"][:, hs]), r.l_out, TOL, f"{tag} L_out")
        del ref


def video_rows(B, tile=128):
    """One row inside every row tile of `tile` rows (a different offset per tile), plus
    the first and last rows."""
    n_tiles = (B + tile - 1) // tile
    rows = {0, B - 1}
    for t in range(n_tiles):
        rows.add(min(B - 1, t * tile + (t * 37 + 5) % tile))
    return np.array(sorted(rows))


def test_video_full_size_every_row_tile(fb):
    w = W.get("video")
    seed = 4
    sched = list(W.block_schedule(w, seed))
    k, v = W.prefix_kv(w, seed)
    got = gpu_replay(fb, w, k, v, sched)
    scale = 1 / math.sqrt(w.head_dim)
    tiles = video_rows(w.block)
    assert len(tiles) >= 37
    full_heads = (0, 7)
    mixed = False
    for h in range(w.h_q):
        kh, vh = k[:, h:h + 1].double().numpy(), v[:, h:h + 1].double().numpy()
        rows = np.arange(w.block) if h in full_heads else tiles
        # rows are independent: the oracle runs on chunks of rows to bound its memory
        chunks = [rows[i:i + 1170] for i in range(0, len(rows), 1170)]
        refs = [OF.CachedBlockAttention(kh, vh, 1, scale) for _ in chunks]
        for s, o in zip(sched, got):
            tag = f"video step {s.index} head {h}"
            M, reuse = OF.decisions(s.mask.numpy(), s.first, w.tau, s.sim.numpy(), w.gamma, w.h_q)
            assert np.array_equal(o["M"], M), f"{tag}: M"
            assert np.array_equal(o["reuse"], reuse), f"{tag}: reuse"
            if 0 < reuse[0].sum() < w.h_q:
                mixed = True
            for rows_c, ref in zip(chunks, refs):
                r = ref.step(f64(s.q[:, h:h + 1, rows_c]), f64(s.k_blk[:, h:h + 1]), f64(s.v_blk[:, h:h + 1]),
                             s.mask.numpy(), s.first, w.tau, s.sim[:, h:h + 1].numpy(), w.gamma)
                assert np.array_equal(r.reuse, reuse[:, h:h + 1])
                close(f64(o["a_full"][:, h:h + 1, rows_c]), r.a_full, TOL, f"{tag} A_full")
                close(f64(o["l_full"][:, h:h + 1, rows_c]), r.l_full, TOL, f"{tag} L_full")
                close(f64(o["a_out"][:, h:h + 1, rows_c]), r.a_out, TOL, f"{tag} A_out")
                close(f64(o["l_out"][:, h:h + 1, rows_c]), r.l_out, TOL, f"{tag} L_out")
    assert mixed, "want steps where some heads reuse and others recompute"
