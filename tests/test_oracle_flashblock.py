"""Pins of oracle.flashblock: gates, the cached step, and the special cases that
reduce to dense attention (CPU only)."""
import json
import os

import numpy as np

from block_diffusion_attention_prefix_b200 import workloads as W
from oracle import attention as OA
from oracle import flashblock as OF

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f64(t):
    return t.to("cpu").double().numpy()


def small(name="tiny_f32", **kw):
    return W.get(name).with_(**kw)


def test_golden_gate_cases():
    data = json.load(open(os.path.join(GOLDEN, "gate_cases.json")))
    for c in data["cases"]:
        B = 8
        mask = np.zeros((1, B), dtype=np.uint8)
        mask[0, :c["M"]] = 1
        sim = None if c["sim"] is None else np.array([[c["sim"]]], dtype=np.float32)
        M, reuse = OF.decisions(mask, c["first"], c["tau"], sim, c["gamma"], 1)
        assert M[0] == c["M"]
        assert bool(reuse[0, 0]) == c["reuse"], c


def replay(w, seed, tau=None, gamma=None, steps=None):
    k, v = W.prefix_kv(w, seed)
    scale = W.default_scale(w.head_dim)
    st = OF.CachedBlockAttention(f64(k), f64(v), w.h_q, scale)
    out = []
    for s in W.block_schedule(w, seed, steps):
        r = st.step(f64(s.q), f64(s.k_blk), f64(s.v_blk), s.mask.numpy(), s.first,
                    w.tau if tau is None else tau,
                    None if s.sim is None else s.sim.numpy(),
                    (w.gamma or 0.0) if gamma is None else gamma)
        dense = OF.dense_attention(f64(s.q), f64(k), f64(v), f64(s.k_blk), f64(s.v_blk), scale)
        out.append((s, r, dense))
    return out


def test_tau_nonpositive_always_recomputes_and_equals_dense():
    w = small(n_prefix=300, h_q=4, h_kv=2, block=5)
    for s, r, (Ad, Ld) in replay(w, 11, tau=0):
        assert not r.reuse.any()
        np.testing.assert_allclose(r.a_full, Ad, rtol=0, atol=1e-12)
        np.testing.assert_allclose(r.l_full, Ld, rtol=0, atol=1e-12)


def test_tau_above_block_reuses_after_first_step():
    w = small(n_prefix=200, block=4)
    res = replay(w, 12, tau=w.block + 1)
    cache0 = res[0][1].a_out
    for s, r, _ in res[1:]:
        assert r.reuse.all()
        np.testing.assert_array_equal(r.a_out, cache0)      # cache untouched


def test_updated_count_and_decision_per_step():
    w = small()
    for s, r, _ in replay(w, 13):
        M = int(s.mask.sum())
        assert r.M[0] == M
        assert bool(r.reuse[0, 0]) == ((not s.first) and M < w.tau)


def test_gamma_extremes():
    w = W.get("video").with_(n_prefix=96, block=24, h_q=3, h_kv=3, head_dim=32)
    # gamma >= every sim: every head recomputes, so every step is dense attention
    for s, r, (Ad, Ld) in replay(w, 14, gamma=1.0):
        assert not r.reuse.any()
        np.testing.assert_allclose(r.a_full, Ad, rtol=0, atol=1e-12)
    # gamma below every sim: every head reuses after step 0
    res = replay(w, 14, gamma=0.5)
    for s, r, _ in res[1:]:
        assert r.reuse.all()
        np.testing.assert_array_equal(r.a_out, res[0][1].a_out)


def test_gamma_per_head_selection_matches_sim():
    w = W.get("video").with_(n_prefix=64, block=16, h_q=6, h_kv=6, head_dim=16)
    res = replay(w, 15)
    prev = None
    for s, r, (Ad, Ld) in res:
        want = np.zeros((1, 6), bool) if s.first else (s.sim.numpy() > np.float32(0.95))
        np.testing.assert_array_equal(r.reuse, want)
        # recomputed heads are exact dense attention
        for h in range(6):
            if not want[0, h]:
                np.testing.assert_allclose(r.a_full[0, h], Ad[0, h], rtol=0, atol=1e-12)
            else:
                np.testing.assert_array_equal(r.a_out[0, h], prev.a_out[0, h])
        prev = r


def test_M_zero_step_reproduces_previous_output_bit_for_bit():
    # with no token updated the inputs are unchanged; a reuse step must give the
    # previous step's A_full exactly and leave the cache untouched
    w = small(n_prefix=128)
    res = replay(w, 0)
    seen = 0
    for (s0, r0, _), (s1, r1, _) in zip(res, res[1:]):
        if int(s1.mask.sum()) == 0:
            seen += 1
            assert r1.reuse.all()
            np.testing.assert_array_equal(r1.a_full, r0.a_full)
            np.testing.assert_array_equal(r1.l_full, r0.l_full)
            np.testing.assert_array_equal(r1.a_out, r0.a_out)
    assert seen >= 1   # the tiny schedule with seed 0 has an M = 0 step (step 5)


def test_reuse_rows_with_unchanged_query_equal_dense():
    # on a reuse step, rows whose query has not changed since the last recompute
    # see a fresh cache, so their output is dense attention over J_out U J_in
    w = small("dlm8b_b4", n_prefix=333, h_q=4, h_kv=2, head_dim=32, block=8, tau=3)
    res = replay(w, 21)
    changed = np.zeros(w.block, dtype=bool)
    checked = 0
    for s, r, (Ad, Ld) in res:
        if not r.reuse[0, 0]:
            changed[:] = False
            np.testing.assert_allclose(r.a_full, Ad, rtol=0, atol=1e-12)
            continue
        changed |= s.mask.numpy()[0].astype(bool)
        for i in np.nonzero(~changed)[0]:
            np.testing.assert_allclose(r.a_full[0, :, i], Ad[0, :, i], rtol=0, atol=1e-12)
            checked += 1
        # and rows whose query did change are not (stale A_out is an approximation)
        for i in np.nonzero(changed)[0]:
            assert np.abs(r.a_full[0, :, i] - Ad[0, :, i]).max() > 1e-9
    assert checked > 0


def test_gqa_head_mapping():
    # query head h reads KV head h // G: permuting KV heads permutes the output blocks
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 4, 3, 8))
    k = rng.standard_normal((1, 2, 50, 8))
    v = rng.standard_normal((1, 2, 50, 8))
    A, L = OF.prefix_attention(q, k, v, 0.3)
    for h in range(4):
        a, l = OA.attend(q[0, h], k[0, h // 2], v[0, h // 2], 0.3)
        np.testing.assert_array_equal(A[0, h], a)
    A2, _ = OF.prefix_attention(q, k[:, ::-1], v[:, ::-1], 0.3)
    assert np.abs(A2[0, 0] - A[0, 0]).max() > 1e-6


def test_updated_count_counts_nonzero_entries():
    # a nonzero mask entry marks an updated token, whatever its value
    mask = np.array([[0, 2, 255, 0], [1, 1, 0, 0], [0, 0, 0, 0]], dtype=np.uint8)
    np.testing.assert_array_equal(OF.updated_count(mask), [2, 2, 0])
