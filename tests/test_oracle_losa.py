"""Pins of oracle.losa (CPU only): LoSA-style per-token reuse.

Pinned by: the library mean of squared differences (numpy) for the locality
score, exact summation (math.fsum), closed forms (delta above every score: every
row reuses its cache, which after a dense first step is the cached FlashBlock step
with reuse; delta below every score with density one: every step is dense attention
with the current queries), and the union over active rows being the union of their
own selections (subset of the union over all rows)."""
import math

import numpy as np

from block_diffusion_attention_prefix_b200 import workloads as W
from oracle import flashblock as OF
from oracle import losa as OL
from oracle import sparse as OS


def test_token_mse_matches_library_mean():
    rng = np.random.default_rng(0)
    q, p = rng.standard_normal((2, 5, 7, 16)), rng.standard_normal((2, 5, 7, 16))
    got = OL.token_mse(q, p)
    want = ((q - p) ** 2).mean(axis=(1, 3)).astype(np.float32)
    np.testing.assert_allclose(got, want, rtol=1e-6)
    for bi in range(2):
        for i in range(7):
            terms = ((q[bi, :, i] - p[bi, :, i]) ** 2).reshape(-1).tolist()
            assert abs(float(got[bi, i]) - math.fsum(terms) / 80) <= 1e-6 * math.fsum(terms) / 80


def test_unchanged_token_scores_zero():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((1, 4, 6, 8))
    p = q.copy()
    p[0, :, 2] += 0.5
    mse = OL.token_mse(q, p)
    assert np.all(mse[0, [0, 1, 3, 4, 5]] == 0.0) and np.isclose(mse[0, 2], 0.25)


def _run(w, seed, delta, density, steps=4):
    k, v = W.prefix_kv(w, seed)
    scale = 1 / math.sqrt(w.head_dim)
    lo = OL.LosaAttention(k.double().numpy(), v.double().numpy(), w.h_q, scale, 16, density)
    prev = None
    out = []
    for s in W.block_schedule(w, seed, steps):
        q = s.q.double().numpy()
        r = lo.step(q, prev, s.k_blk.double().numpy(), s.v_blk.double().numpy(), s.first, delta)
        out.append((s, r))
        prev = q
    return k, v, out


W_SMALL = W.get("sparse64k").with_(n_prefix=300, h_q=4, h_kv=2, head_dim=16, block=6)


def test_delta_above_every_score_reuses_the_cache():
    k, v, out = _run(W_SMALL, 2, 1e30, 0.3)
    ref = OF.CachedBlockAttention(k.double().numpy(), v.double().numpy(), W_SMALL.h_q, 1 / math.sqrt(16))
    for s, r in out:
        rf = ref.step(s.q.double().numpy(), s.k_blk.double().numpy(), s.v_blk.double().numpy(), s.mask.numpy(),
                      s.first, W_SMALL.block + 1)   # tau = B + 1: reuse after the first step
        assert not r.active.any() or s.first
        np.testing.assert_array_equal(r.a_full, rf.a_full)
        np.testing.assert_array_equal(r.l_full, rf.l_full)


def test_all_active_with_density_one_is_dense():
    k, v, out = _run(W_SMALL, 3, -1.0, 1.0)
    for s, r in out:
        Ad, Ld = OF.dense_attention(s.q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                    s.k_blk.double().numpy(), s.v_blk.double().numpy(), 1 / math.sqrt(16))
        np.testing.assert_allclose(r.a_full, Ad, atol=1e-12)
        np.testing.assert_allclose(r.l_full, Ld, atol=1e-12)


def test_union_is_over_active_rows_only():
    k, v, out = _run(W_SMALL.with_(n_prefix=2000), 4, 1e-3, 0.2, steps=5)
    some_stable = False
    for s, r in out[1:]:
        G = W_SMALL.h_q // W_SMALL.h_kv
        for g in range(W_SMALL.h_kv):
            rows = r.sel[0, g * G:(g + 1) * G]
            act = rows[:, r.active[0]].reshape(-1)
            P = OS.n_pages(2000, 16)
            np.testing.assert_array_equal(r.union[0, g], OS.union_bitmap(act, P))
            assert np.all(rows[:, ~r.active[0]] == -1)
        some_stable |= bool((~r.active).any()) and bool(r.active.any())
    assert some_stable, "want steps with both active and stable tokens"


def test_delta_zero_keeps_unmoved_tokens_stable():
    # tokens not updated keep their queries bit for bit, so their score is exactly 0;
    # with delta = 0 the strict comparison keeps them stable and only moved tokens
    # are active
    k, v, out = _run(W_SMALL, 5, 0.0, 0.2, steps=6)
    mixed = 0
    for s, r in out[1:]:
        moved = s.mask.numpy()[0].astype(bool)
        np.testing.assert_array_equal(r.active[0], moved)
        mixed += bool(moved.any()) and bool((~moved).any())
    assert mixed > 0
