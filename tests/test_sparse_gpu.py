"""GPU parity of the sparse-residual mode (page bounds, top-k selection, residual
cache, sparse step) against the CPU oracle (oracle.sparse).

Integer outputs -- page selections, row bitmaps, the union bitmap of each KV
group, M and the reuse decisions -- must match bit for bit; floating outputs
within the bf16 tolerance 2e-2.
"""
import math

import numpy as np
import pytest
import torch

from block_diffusion_attention_prefix_b200 import workloads as W
from oracle import flashblock as OF
from oracle import sparse as OS

pytestmark = pytest.mark.gpu
TOL = 2e-2


def f64(t):
    return t.detach().to("cpu").double().numpy()


def close(got, want, tol, what=""):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(want)), f"{what}: -inf pattern differs"
    m = ~np.isneginf(want)
    err = np.abs(got[m] - want[m]).max() if m.any() else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


def bits_to_pages(words, n_pages):
    w = np.asarray(words).astype(np.uint32)
    out = []
    for p in range(n_pages):
        if (int(w[p // 32]) >> (p % 32)) & 1:
            out.append(p)
    return np.array(out, dtype=np.int64)


@pytest.mark.parametrize("N", [16, 1000, 4096, 5003])
def test_page_minmax_exact(fb, N):
    g = torch.Generator().manual_seed(N)
    k = torch.randn((2, 3, N, 128), generator=g).to(torch.bfloat16)
    sh = fb.make_shape(2, 6, 3, 128, 4, N, "bf16")
    P = (N + 15) // 16
    kmin = torch.empty((2, 3, 128, fb.fb_page_cap(sh)), dtype=torch.bfloat16, device="cuda")
    kmax = torch.empty_like(kmin)
    fb.fb_page_minmax(sh, k.cuda(), 16, kmin, kmax)
    for bi in range(2):
        for g_ in range(3):
            mn, mx = OS.page_minmax(f64(k[bi, g_]), 16)
            assert np.array_equal(f64(kmin[bi, g_, :, :P]).T, mn)
            assert np.array_equal(f64(kmax[bi, g_, :, :P]).T, mx)


def select_case(fb, w, seed, tie_pages=False):
    k, v = W.prefix_kv(w, seed)
    if tie_pages:  # duplicate pages 0..3 into 4..7 and 10..13: identical bounds, tied estimates
        k[:, :, 64:128] = k[:, :, 0:64]
        k[:, :, 160:224] = k[:, :, 0:64]
    s = next(iter(W.block_schedule(w, seed, 1)))
    n_sel = OS.n_selected(w.n_prefix, 16, w.density)
    layer = fb.SparseResidualLayer(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, k.cuda(), v.cuda(), n_sel)
    gate = fb.make_gate(s.mask.cuda(), True, w.tau)
    fb.fb_sparse_select(layer.shape, s.q.cuda(), gate, layer.sparse, layer.ws)
    torch.cuda.synchronize()
    q = f64(s.q)
    P = layer.n_pages
    for bi in range(w.batch):
        for h in range(w.h_q):
            kmin, kmax = OS.page_minmax(f64(k[bi, h // w.group]), 16)
            est = OS.page_estimates(q[bi, h], kmin, kmax)
            want = OS.select_pages(est, n_sel)
            got = layer.sel_idx[bi, h].cpu().numpy()
            assert np.array_equal(got, want), f"selection differs at b={bi} h={h}"
            for i in range(w.block):
                assert np.array_equal(bits_to_pages(layer.sel_bits[bi, h, i].cpu().numpy(), P), want[i])
        for g_ in range(w.h_kv):
            rows = layer.sel_idx[bi, g_ * w.group:(g_ + 1) * w.group].cpu().numpy().reshape(-1)
            want_u = OS.union_bitmap(rows, P)
            assert np.array_equal(layer.union_bits[bi, g_].cpu().numpy().astype(np.uint32), want_u)
    return layer


SMALL = W.get("sparse64k").with_(n_prefix=3000, h_q=8, h_kv=2, steps=6)


def test_select_bit_exact(fb):
    select_case(fb, SMALL, 1)


def test_select_ties_go_to_lower_pages(fb):
    select_case(fb, SMALL.with_(density=0.1), 2, tie_pages=True)


def test_select_density_extremes(fb):
    select_case(fb, SMALL.with_(density=1.0), 3)
    select_case(fb, SMALL.with_(density=0.001), 4)


def replay_sparse(fb, w, seed, density=None, check_sel=True):
    density = w.density if density is None else density
    k, v = W.prefix_kv(w, seed)
    n_sel = OS.n_selected(w.n_prefix, 16, density)
    layer = fb.SparseResidualLayer(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, k.cuda(), v.cuda(), n_sel,
                                   keep_sel=True)
    ref = OS.SparseResidualAttention(f64(k), f64(v), w.h_q, 1 / math.sqrt(w.head_dim), 16, density)
    out = []
    for s in W.block_schedule(w, seed):
        layer.step(s.q.cuda(), s.k_blk.cuda(), s.v_blk.cuda(), s.mask.cuda(), s.first, w.tau)
        r = ref.step(f64(s.q), f64(s.k_blk), f64(s.v_blk), s.mask.numpy(), s.first, w.tau)
        torch.cuda.synchronize()
        assert np.array_equal(layer.dec_M.cpu().numpy(), r.M), f"step {s.index} M"
        assert np.array_equal(layer.dec_reuse.cpu().numpy().astype(bool), r.reuse), f"step {s.index} reuse"
        if check_sel:
            assert np.array_equal(layer.sel_idx.cpu().numpy(), r.sel), f"step {s.index} selection"
            assert np.array_equal(layer.union_bits.cpu().numpy().astype(np.uint32), r.union), f"step {s.index} union"
        close(f64(layer.a_res), r.a_res, TOL, f"step {s.index} A_res")
        close(f64(layer.l_res), r.l_res, TOL, f"step {s.index} L_res")
        close(f64(layer.a_sel), r.a_sel, TOL, f"step {s.index} A_sel")
        close(f64(layer.l_sel), r.l_sel, TOL, f"step {s.index} L_sel")
        close(f64(layer.a_full), r.a_full, TOL, f"step {s.index} A_full")
        close(f64(layer.l_full), r.l_full, TOL, f"step {s.index} L_full")
        out.append((s, r))
    assert fb.fb_device_error() == 0
    return layer, out


def test_sparse_schedule_small(fb):
    _, out = replay_sparse(fb, SMALL, 5)
    assert {bool(r.reuse.any()) for _, r in out} == {True, False}


def test_sparse_schedule_ragged_prefix_and_block16(fb):
    w = SMALL.with_(n_prefix=2011, block=8, tau=3, h_q=8, h_kv=2)  # R = 32 rows, partial last page
    replay_sparse(fb, w, 6)


def test_sparse_density_one_is_dense(fb):
    w = SMALL.with_(steps=3)
    layer, out = replay_sparse(fb, w, 7, density=1.0)
    assert torch.isneginf(layer.l_res).all()
    k, v = W.prefix_kv(w, 7)
    s, r = out[0]
    Ad, Ld = OF.dense_attention(f64(s.q), f64(k), f64(v), f64(s.k_blk), f64(s.v_blk), 1 / math.sqrt(w.head_dim))
    close(r.a_full, Ad, 1e-9, "oracle")


def test_sparse_full_size_schedule(fb):
    """The sparse workload at full size: N = 65536 (4096 pages), 820 pages per
    query row, 32 query heads / 8 KV heads, 16 steps."""
    layer, out = replay_sparse(fb, W.get("sparse64k"), 8)
    u = layer.union_bits.cpu().numpy().astype(np.uint32)
    density = np.mean([bin(int(x)).count("1") for x in u.reshape(-1)]) / 32
    assert 0.5 < density <= 1.0   # KV inflation: the union over 16 rows covers most pages
