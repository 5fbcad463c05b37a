"""GPU parity of the block transition (fb_append_block) and of multi-block
generation against the CPU oracle (oracle.transition).

The append is a copy, so it is checked bit for bit (rows before and after the new
ones untouched); the refreshed page bounds bit for bit; generation schedules
within the dtype tolerances (fp32 1e-5, bf16 2e-2) with decisions and sparse
selections bit-exact.
"""
import math

import numpy as np
import pytest
import torch

from block_diffusion_attention_prefix_b200 import workloads as W
from oracle import flashblock as OF
from oracle import sparse as OS
from oracle import transition as OT

pytestmark = pytest.mark.gpu
TOL = {"f32": 1e-5, "bf16": 2e-2}


def f64(t):
    return t.detach().to("cpu").double().numpy()


def close(got, want, tol, what=""):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(want)), f"{what}: -inf pattern differs"
    m = ~np.isneginf(want)
    err = np.abs(got[m] - want[m]).max() if m.any() else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


def cache_with_room(b, hkv, N, cap, D, rs, dtype, seed):
    """K/V caches [b, hkv, cap, rs] (row stride rs >= D): N random rows, the rest a sentinel."""
    g = torch.Generator().manual_seed(seed)
    k = torch.full((b, hkv, cap, rs), 3.0).to(dtype)
    v = torch.full((b, hkv, cap, rs), -3.0).to(dtype)
    k[:, :, :N, :D] = torch.randn((b, hkv, N, D), generator=g).to(dtype)
    v[:, :, :N, :D] = torch.randn((b, hkv, N, D), generator=g).to(dtype)
    return k, v


@pytest.mark.parametrize("dtype,D,rs", [("bf16", 128, 128), ("bf16", 64, 96), ("f32", 64, 64), ("f32", 128, 136)])
@pytest.mark.parametrize("N,B", [(0, 4), (15, 16), (1000, 37)])
def test_append_block_copies_rows(fb, dtype, D, rs, N, B):
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    b, hkv, cap = 2, 3, N + B + 5
    k, v = cache_with_room(b, hkv, N, cap, D, rs, td, N + B)
    g = torch.Generator().manual_seed(7)
    kb = torch.randn((b, hkv, B, D), generator=g).to(td)
    vb = torch.randn((b, hkv, B, D), generator=g).to(td)
    kd, vd = k.cuda(), v.cuda()
    sh = fb.make_shape(b, 4 * hkv, hkv, D, B, N, dtype, kv_row_stride=rs, kv_head_stride=cap * rs)
    fb.fb_append_block(sh, kd, vd, kb.cuda(), vb.cuda())
    torch.cuda.synchronize()
    kw, vw = k.clone(), v.clone()
    kw[:, :, N:N + B, :D] = kb
    vw[:, :, N:N + B, :D] = vb
    assert torch.equal(kd.cpu(), kw) and torch.equal(vd.cpu(), vw)


@pytest.mark.parametrize("N,B", [(15, 4), (16, 16), (17, 37), (1000, 16), (2000, 64)])
def test_append_block_refreshes_touched_page_bounds(fb, N, B):
    b, hkv, D, cap = 1, 2, 128, N + B + 40
    k, v = cache_with_room(b, hkv, N, cap, D, D, torch.bfloat16, N)
    g = torch.Generator().manual_seed(9)
    kb = torch.randn((b, hkv, B, D), generator=g).to(torch.bfloat16)
    vb = torch.randn((b, hkv, B, D), generator=g).to(torch.bfloat16)
    kd, vd = k.cuda(), v.cuda()
    sh = fb.make_shape(b, 4 * hkv, hkv, D, B, N, "bf16", kv_head_stride=cap * D)
    page_cap = fb.fb_page_cap(sh)
    assert page_cap == ((cap + 15) // 16 + 7) // 8 * 8
    kmin = torch.full((b, hkv, D, page_cap), 5.0, dtype=torch.bfloat16, device="cuda")
    kmax = kmin.clone()
    fb.fb_page_minmax(sh, kd, 16, kmin, kmax)
    fb.fb_append_block(sh, kd, vd, kb.cuda(), vb.cuda(), 16, kmin, kmax)
    torch.cuda.synchronize()
    P = OS.n_pages(N + B, 16)
    for g_ in range(hkv):
        old_min, old_max = OS.page_minmax(f64(k[0, g_, :N]), 16)
        grown = np.concatenate([f64(k[0, g_, :N]), f64(kb[0, g_])])
        want_min, want_max = OT.update_page_minmax(old_min, old_max, grown, N, 16)
        assert np.array_equal(f64(kmin[0, g_, :, :P]).T, want_min)
        assert np.array_equal(f64(kmax[0, g_, :, :P]).T, want_max)
        assert bool((kmin[0, g_, :, P:] == 5.0).all()) and bool((kmax[0, g_, :, P:] == 5.0).all())


def test_append_block_rejects_a_cache_without_room(fb):
    b, hkv, D, N, B = 1, 2, 64, 100, 8
    k = torch.zeros((b, hkv, N + B, D), dtype=torch.bfloat16, device="cuda")
    kb = torch.zeros((b, hkv, B, D), dtype=torch.bfloat16, device="cuda")
    for head_stride in ((N + B - 1) * D, 0):  # one row short; contiguous (no room at all)
        sh = fb.make_shape(b, hkv, hkv, D, B, N, "bf16", kv_head_stride=head_stride)
        with pytest.raises(fb.FBError) as ei:
            fb.fb_append_block(sh, k, k, kb, kb)
        assert ei.value.status == -2
    assert bool((k == 0).all())


def run_generation(fb, w, seed, blocks, steps):
    """Dense generation: blocks x steps through fb_step and fb_append_block vs the oracle."""
    k, v = W.prefix_kv(w, seed)
    cap = w.n_prefix + blocks * w.block
    kc = torch.zeros((w.batch, w.h_kv, cap, w.head_dim), dtype=w.torch_dtype)
    vc = torch.zeros_like(kc)
    kc[:, :, :w.n_prefix], vc[:, :, :w.n_prefix] = k, v
    layer = fb.CachedAttentionLayer(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, kc.cuda(), vc.cuda(),
                                    n_prefix=w.n_prefix)
    ref = OF.CachedBlockAttention(f64(k), f64(v), w.h_q, 1 / math.sqrt(w.head_dim))
    tol = TOL[w.dtype]
    for t, block in enumerate(W.generation_schedule(w, seed, blocks, steps)):
        for s in block:
            layer.step(s.q.cuda(), s.k_blk.cuda(), s.v_blk.cuda(), s.mask.cuda(), s.first, w.tau)
            r = ref.step(f64(s.q), f64(s.k_blk), f64(s.v_blk), s.mask.numpy(), s.first, w.tau)
            torch.cuda.synchronize()
            what = f"block {t} step {s.index}"
            assert np.array_equal(layer.dec_reuse.cpu().numpy().astype(bool), r.reuse), what
            close(f64(layer.a_full), r.a_full, tol, what + " A_full")
            close(f64(layer.l_full), r.l_full, tol, what + " L_full")
            close(f64(layer.a_out), r.a_out, tol, what + " A_out")
        layer.finish_block(block[-1].k_blk.cuda(), block[-1].v_blk.cuda())
        ref.finish_block(f64(block[-1].k_blk), f64(block[-1].v_blk))
        assert layer.shape.n_prefix == w.n_prefix + (t + 1) * w.block
    assert fb.fb_device_error() == 0


@pytest.mark.parametrize("name,kw", [
    ("dlm8b_b4", dict(n_prefix=1000)),              # 16 rows per KV head: mma.sync pass
    ("dlm8b_b16", dict(n_prefix=1500, tau=5)),      # 64 rows per KV head: tcgen05 split pass
    ("tiny_f32", dict(n_prefix=300, block=7)),      # fp32, ragged pages and tiles
])
def test_generation_dense(fb, name, kw):
    run_generation(fb, W.get(name).with_(**kw), seed=21, blocks=3, steps=4)


def test_generation_sparse(fb):
    w = W.get("sparse64k").with_(n_prefix=3000, h_q=8, h_kv=2, block=8, tau=3)
    seed, blocks, steps = 22, 3, 4
    k, v = W.prefix_kv(w, seed)
    cap = w.n_prefix + blocks * w.block
    kc = torch.zeros((w.batch, w.h_kv, cap, w.head_dim), dtype=w.torch_dtype)
    vc = torch.zeros_like(kc)
    kc[:, :, :w.n_prefix], vc[:, :, :w.n_prefix] = k, v
    n_sel = OS.n_selected(w.n_prefix, 16, w.density)
    layer = fb.SparseResidualLayer(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, kc.cuda(), vc.cuda(), n_sel,
                                   keep_sel=True, n_prefix=w.n_prefix)
    ref = OS.SparseResidualAttention(f64(k), f64(v), w.h_q, 1 / math.sqrt(w.head_dim), 16, w.density)
    for t, block in enumerate(W.generation_schedule(w, seed, blocks, steps)):
        for s in block:
            layer.step(s.q.cuda(), s.k_blk.cuda(), s.v_blk.cuda(), s.mask.cuda(), s.first, w.tau)
            r = ref.step(f64(s.q), f64(s.k_blk), f64(s.v_blk), s.mask.numpy(), s.first, w.tau)
            torch.cuda.synchronize()
            what = f"block {t} step {s.index}"
            assert np.array_equal(layer.dec_reuse.cpu().numpy().astype(bool), r.reuse), what
            assert np.array_equal(layer.sel_idx.cpu().numpy(), r.sel), what + " selection"
            assert np.array_equal(layer.union_bits.cpu().numpy().astype(np.uint32), r.union), what + " union"
            close(f64(layer.a_full), r.a_full, 2e-2, what + " A_full")
            close(f64(layer.a_res), r.a_res, 2e-2, what + " A_res")
        layer.finish_block(block[-1].k_blk.cuda(), block[-1].v_blk.cuda(),
                           OS.n_selected(w.n_prefix + (t + 1) * w.block, 16, w.density))
        ref.finish_block(f64(block[-1].k_blk), f64(block[-1].v_blk))
        assert layer.sparse.n_select == ref.k_sel
    assert fb.fb_device_error() == 0
