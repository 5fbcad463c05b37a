"""Pins of oracle.sparse: page bounds, top-k selection, residual split (CPU only)."""
import math

import numpy as np
import pytest

from block_diffusion_attention_prefix_b200 import workloads as W
from oracle import attention as OA
from oracle import flashblock as OF
from oracle import sparse as OS


def bf16_grid(rng, shape, scale=1.0):
    # values exactly representable in bf16 (8 significant bits)
    x = rng.standard_normal(shape) * scale
    e = np.floor(np.log2(np.abs(x) + 1e-300))
    return np.round(x / 2.0 ** (e - 7)) * 2.0 ** (e - 7)


def test_page_minmax_partial_last_page():
    rng = np.random.default_rng(0)
    k = rng.standard_normal((37, 5))
    kmin, kmax = OS.page_minmax(k, 16)
    assert kmin.shape == (3, 5)
    np.testing.assert_array_equal(kmin[2], k[32:37].min(0))
    np.testing.assert_array_equal(kmax[2], k[32:37].max(0))


def test_page_estimate_bounds_every_score_in_page():
    rng = np.random.default_rng(1)
    k = bf16_grid(rng, (203, 16))
    q = bf16_grid(rng, (6, 16))
    kmin, kmax = OS.page_minmax(k, 16)
    est = OS.page_estimates(q, kmin, kmax)
    s = q @ k.T
    for p in range(kmin.shape[0]):
        page_max = s[:, p * 16:min(203, (p + 1) * 16)].max(axis=1)
        assert np.all(est[:, p] >= page_max - 1e-12)


def test_page_estimate_single_token_page_is_exact_score():
    # with one token per page kmin = kmax = k, so the bound is q . k exactly
    rng = np.random.default_rng(2)
    k = bf16_grid(rng, (20, 8))
    q = bf16_grid(rng, (3, 8))
    kmin, kmax = OS.page_minmax(k, 1)
    est = OS.page_estimates(q, kmin, kmax)
    exact = np.array([[math.fsum(float(a) * float(b) for a, b in zip(qq, kk)) for kk in k] for qq in q])
    np.testing.assert_allclose(est, exact, rtol=0, atol=1e-12)


def test_page_estimate_is_ordered_float64_sum():
    # the estimate is the left-to-right float64 sum over d, term by term
    rng = np.random.default_rng(3)
    kmin = bf16_grid(rng, (7, 12))
    kmax = kmin + np.abs(bf16_grid(rng, (7, 12)))
    q = bf16_grid(rng, (2, 12))
    est = OS.page_estimates(q, kmin, kmax)
    for r in range(2):
        for p in range(7):
            acc = 0.0
            for d in range(12):
                acc = acc + max(q[r, d] * kmin[p, d], q[r, d] * kmax[p, d])
            assert est[r, p] == acc


@pytest.mark.parametrize("seed", range(4))
def test_select_pages_matches_full_lexsort(seed):
    rng = np.random.default_rng(seed)
    est = np.round(rng.standard_normal((5, 300)), 1)      # many ties
    k = int(rng.integers(1, 300))
    sel = OS.select_pages(est, k)
    for r in range(5):
        order = np.lexsort((np.arange(300), -est[r]))     # library sort, index tie-break
        np.testing.assert_array_equal(sel[r], np.sort(order[:k]))


def test_select_ties_prefer_lower_page():
    est = np.array([[1.0, 2.0, 2.0, 2.0, 0.5]])
    np.testing.assert_array_equal(OS.select_pages(est, 2), [[1, 2]])
    np.testing.assert_array_equal(OS.select_pages(est, 4), [[0, 1, 2, 3]])


def test_n_selected():
    assert OS.n_selected(65536, 16, 0.2) == 820
    assert OS.n_selected(100, 16, 0.2) == 2          # 7 pages, ceil(1.4)
    assert OS.n_selected(100, 16, 1.0) == 7
    assert OS.n_selected(10, 16, 0.01) == 1


def test_union_bitmap():
    sel = np.array([[0, 5, 33], [5, 63, 64]])
    words = OS.union_bitmap(sel, 65)
    assert words.tolist() == [(1 << 0) | (1 << 5), (1 << 1) | (1 << 31), 1]


def f64(t):
    return t.double().numpy()


def replay_sparse(w, seed, **kw):
    k, v = W.prefix_kv(w, seed)
    scale = W.default_scale(w.head_dim)
    st = OS.SparseResidualAttention(f64(k), f64(v), w.h_q, scale, w.page_size, kw.get("density", w.density))
    for s in W.block_schedule(w, seed):
        r = st.step(f64(s.q), f64(s.k_blk), f64(s.v_blk), s.mask.numpy(), s.first, kw.get("tau", w.tau))
        d = OF.dense_attention(f64(s.q), f64(k), f64(v), f64(s.k_blk), f64(s.v_blk), scale)
        yield s, r, d


SMALL = W.get("sparse64k").with_(n_prefix=300, h_q=4, h_kv=2, head_dim=16, block=4, steps=6)


def test_density_one_leaves_empty_residual_and_equals_dense():
    for s, r, (Ad, Ld) in replay_sparse(SMALL, 1, density=1.0):
        assert np.all(np.isneginf(r.l_res))
        np.testing.assert_allclose(r.a_full, Ad, rtol=0, atol=1e-12)


def test_recompute_step_equals_dense_and_selection_is_frozen_on_reuse():
    prev = None
    n_reuse = 0
    for s, r, (Ad, Ld) in replay_sparse(SMALL, 2):
        if not r.reuse.any():
            np.testing.assert_allclose(r.a_full, Ad, rtol=0, atol=1e-12)
            np.testing.assert_allclose(r.l_full, Ld, rtol=0, atol=1e-12)
        else:
            n_reuse += 1
            np.testing.assert_array_equal(r.sel, prev.sel)
            np.testing.assert_array_equal(r.a_res, prev.a_res)
        # selected + residual partition the prefix: their key sets are disjoint and cover it
        assert r.sel.shape[-1] == OS.n_selected(300, 16, 0.2)
        prev = r
    assert n_reuse > 0


def test_selected_part_is_attention_over_selected_pages():
    for s, r, _ in replay_sparse(SMALL, 3):
        k, v = W.prefix_kv(SMALL, 3)
        q = f64(s.q)
        for h in (0, 3):
            g = h // 2
            keep = OS.key_mask_from_pages(r.sel[0, h], 300, 16)
            a, l = OA.attend(q[0, h, 1:2], f64(k)[0, g][keep[1]], f64(v)[0, g][keep[1]], W.default_scale(16))
            np.testing.assert_allclose(r.a_sel[0, h, 1], a[0], rtol=0, atol=1e-12)
        break


def test_page_minmax_partial_page_ignores_missing_rows():
    # the last page holds 5 real rows; rows past the prefix must not enter its bounds
    rng = np.random.default_rng(4)
    pos = 1.0 + np.abs(rng.standard_normal((37, 6)))
    kmin, kmax = OS.page_minmax(pos, 16)
    np.testing.assert_array_equal(kmin[2], pos[32:].min(0))
    assert (kmin >= 1.0).all()
    kmin, kmax = OS.page_minmax(-pos, 16)
    np.testing.assert_array_equal(kmax[2], (-pos)[32:].max(0))
    assert (kmax <= -1.0).all()
