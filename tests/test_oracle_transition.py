"""Pins of oracle.transition and of the multi-block generation loop (CPU only).

The block transition appends a finished block's K/V to the prefix (FlashBlock
technical summary, "1. Problem definition": J_out is the earlier blocks).  Pinned
by: the library's softmax attention over the concatenated keys (torch float64
SDPA), the merge identity over the two key sets, page bounds recomputed from
scratch, and dense attention at every block's first step.
"""
import math

import numpy as np
import pytest
import torch

from block_diffusion_attention_prefix_b200 import workloads as W
from oracle import attention as OA
from oracle import flashblock as OF
from oracle import sparse as OS
from oracle import transition as OT


def sdpa(q, k, v, scale):
    """Library softmax attention (torch float64) of q [R, D] over k, v [N, D]: (A, L)."""
    qt, kt, vt = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v))
    A = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None], scale=scale)[0]
    L = torch.logsumexp(scale * qt @ kt.T, dim=1)
    return A.numpy(), L.numpy()


@pytest.mark.parametrize("N,B", [(1, 1), (37, 5), (64, 16), (100, 37)])
def test_appended_prefix_is_old_prefix_then_block(N, B):
    rng = np.random.default_rng(N * 100 + B)
    k, v = rng.standard_normal((2, 3, N, 8)), rng.standard_normal((2, 3, N, 8))
    kb, vb = rng.standard_normal((2, 3, B, 8)), rng.standard_normal((2, 3, B, 8))
    k2, v2 = OT.append_block(k, v, kb, vb)
    assert k2.shape == (2, 3, N + B, 8)
    np.testing.assert_array_equal(k2[:, :, :N], k)
    np.testing.assert_array_equal(k2[:, :, N:], kb)
    np.testing.assert_array_equal(v2[:, :, N:], vb)
    # attention over the grown prefix = library attention over the concatenated keys
    # = the merge of the two key sets (the pages' merge equation)
    q = rng.standard_normal((4, 8))
    scale = 1 / math.sqrt(8)
    A, L = OA.attend(q, k2[1, 2], v2[1, 2], scale)
    At, Lt = sdpa(q, k2[1, 2], v2[1, 2], scale)
    np.testing.assert_allclose(A, At, atol=1e-12)
    np.testing.assert_allclose(L, Lt, atol=1e-12)
    Am, Lm = OA.merge(*OA.attend(q, k[1, 2], v[1, 2], scale), *OA.attend(q, kb[1, 2], vb[1, 2], scale))
    np.testing.assert_allclose(Am, At, atol=1e-12)
    np.testing.assert_allclose(Lm, Lt, atol=1e-12)


@pytest.mark.parametrize("N", [1, 15, 16, 17, 33, 100])
@pytest.mark.parametrize("B", [1, 4, 16, 37])
def test_incremental_page_bounds_equal_recomputed(N, B):
    rng = np.random.default_rng(N * 7 + B)
    k = rng.standard_normal((N, 6))
    kb = rng.standard_normal((B, 6))
    kmin, kmax = OS.page_minmax(k, 16)
    grown = np.concatenate([k, kb])
    umin, umax = OT.update_page_minmax(kmin, kmax, grown, N, 16)
    fmin, fmax = OS.page_minmax(grown, 16)
    np.testing.assert_array_equal(umin, fmin)
    np.testing.assert_array_equal(umax, fmax)


def _dense_reference(q, k_all, v_all, kb, vb, scale):
    b, hq, B, D = q.shape
    G = hq // k_all.shape[1]
    A = np.zeros((b, hq, B, D))
    for bi in range(b):
        for h in range(hq):
            keys = np.concatenate([k_all[bi, h // G], kb[bi, h // G]])
            vals = np.concatenate([v_all[bi, h // G], vb[bi, h // G]])
            A[bi, h] = sdpa(q[bi, h], keys, vals, scale)[0]
    return A


def test_generation_first_steps_are_dense_over_all_earlier_blocks():
    w = W.get("tiny_f32").with_(n_prefix=50, block=6, h_q=4, h_kv=2, steps=3)
    k, v = W.prefix_kv(w, 3)
    k_all, v_all = k.double().numpy(), v.double().numpy()
    scale = 1 / math.sqrt(w.head_dim)
    layer = OF.CachedBlockAttention(k_all, v_all, w.h_q, scale)
    blocks = W.generation_schedule(w, 3, 3)
    for t, steps in enumerate(blocks):
        for s in steps:
            r = layer.step(s.q.double().numpy(), s.k_blk.double().numpy(), s.v_blk.double().numpy(),
                           s.mask.numpy(), s.first, w.tau)
            if s.first:
                want = _dense_reference(s.q.double().numpy(), k_all, v_all, s.k_blk.double().numpy(),
                                        s.v_blk.double().numpy(), scale)
                np.testing.assert_allclose(r.a_full, want, atol=1e-12)
        last = steps[-1]
        layer.finish_block(last.k_blk.double().numpy(), last.v_blk.double().numpy())
        k_all = np.concatenate([k_all, last.k_blk.double().numpy()], axis=2)
        v_all = np.concatenate([v_all, last.v_blk.double().numpy()], axis=2)
        assert layer.k.shape[2] == w.n_prefix + (t + 1) * w.block


def test_sparse_generation_bounds_and_density_one():
    w = W.get("sparse64k").with_(n_prefix=70, block=5, h_q=4, h_kv=2, head_dim=16, steps=2)
    k, v = W.prefix_kv(w, 4)
    scale = 1 / math.sqrt(w.head_dim)
    sp = OS.SparseResidualAttention(k.double().numpy(), v.double().numpy(), w.h_q, scale, 16, 1.0)
    k_all, v_all = k.double().numpy(), v.double().numpy()
    for steps in W.generation_schedule(w, 4, 3):
        for s in steps:
            q, kb, vb = s.q.double().numpy(), s.k_blk.double().numpy(), s.v_blk.double().numpy()
            rs = sp.step(q, kb, vb, s.mask.numpy(), s.first, w.tau)
            # density 1: every page is selected and computed fresh each step, the
            # residual is empty, so every step is dense attention over the grown prefix
            np.testing.assert_allclose(rs.a_full, _dense_reference(q, k_all, v_all, kb, vb, scale), atol=1e-12)
            assert np.all(np.isneginf(rs.l_res))
        last = steps[-1]
        sp.finish_block(last.k_blk.double().numpy(), last.v_blk.double().numpy())
        k_all = np.concatenate([k_all, last.k_blk.double().numpy()], axis=2)
        v_all = np.concatenate([v_all, last.v_blk.double().numpy()], axis=2)
        for bi in range(w.batch):
            for g in range(w.h_kv):
                fmin, fmax = OS.page_minmax(sp.k[bi, g], 16)
                np.testing.assert_array_equal(sp.bounds[bi][g][0], fmin)
                np.testing.assert_array_equal(sp.bounds[bi][g][1], fmax)
        assert sp.k_sel == OS.n_pages(sp.N, 16)
