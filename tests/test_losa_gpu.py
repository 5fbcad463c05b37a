"""GPU parity of the LoSA-style step (fb_losa_step) against the CPU oracle
(oracle.losa): locality scores (float32) and token activity bit for bit, the
selections of active rows and the union over active rows bit for bit, the cache
rows and A_full within the bf16 tolerance 2e-2."""
import math

import numpy as np
import pytest
import torch

from block_diffusion_attention_prefix_b200 import workloads as W
from oracle import losa as OL
from oracle import sparse as OS

pytestmark = pytest.mark.gpu
TOL = 2e-2


def f64(t):
    return t.detach().to("cpu").double().numpy()


def close(got, want, tol, what):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(want)), f"{what}: -inf pattern differs"
    m = ~np.isneginf(want)
    err = np.abs(got[m] - want[m]).max() if m.any() else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e}"


def run(fb, w, seed, delta, steps=None):
    k, v = W.prefix_kv(w, seed)
    n_sel = OS.n_selected(w.n_prefix, 16, w.density)
    layer = fb.LosaLayer(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, k.cuda(), v.cuda(), n_sel, delta,
                         keep_sel=True)
    ref = OL.LosaAttention(f64(k), f64(v), w.h_q, 1 / math.sqrt(w.head_dim), 16, w.density)
    prev = None
    stats = []
    for s in W.block_schedule(w, seed, steps):
        layer.step(s.q.cuda(), s.k_blk.cuda(), s.v_blk.cuda(), s.mask.cuda(), s.first)
        r = ref.step(f64(s.q), prev, f64(s.k_blk), f64(s.v_blk), s.first, delta)
        prev = f64(s.q)
        torch.cuda.synchronize()
        what = f"step {s.index}"
        if not s.first:
            assert np.array_equal(layer.mse.cpu().numpy(), r.mse), what + " score"
            act = layer.active.cpu().numpy().astype(bool)
            assert np.array_equal(act, r.active), what + " activity"
            sel = layer.sel_idx.cpu().numpy()
            for bi in range(w.batch):
                rows = np.nonzero(r.active[bi])[0]
                assert np.array_equal(sel[bi][:, rows], r.sel[bi][:, rows]), what + " selection"
            assert np.array_equal(layer.union_bits.cpu().numpy().astype(np.uint32), r.union), what + " union"
            stats.append((int(r.active.sum()), r.union))
        close(f64(layer.a_res), r.a_out, TOL, what + " cache A")
        close(f64(layer.l_res), r.l_out, TOL, what + " cache L")
        close(f64(layer.a_full), r.a_full, TOL, what + " A_full")
        close(f64(layer.l_full), r.l_full, TOL, what + " L_full")
    assert fb.fb_device_error() == 0
    return stats


def test_token_score_bit_exact(fb):
    # 32 tokens, 8 query heads on 8 KV heads (32 rows per KV head, the sparse kernels' limit)
    g = torch.Generator().manual_seed(3)
    q = torch.randn((2, 8, 32, 128), generator=g).to(torch.bfloat16)
    qp = q.clone()
    qp[:, :, ::3] = torch.randn(qp[:, :, ::3].shape, generator=g).to(torch.bfloat16)
    qp[1, :, 5] = (q[1, :, 5].float() * 1e20).to(torch.bfloat16)  # wide exponent gaps: rounded differences
    w = W.get("sparse64k").with_(n_prefix=64, h_q=8, h_kv=8, block=32, batch=2)
    k, v = W.prefix_kv(w, 3)
    layer = fb.LosaLayer(2, 8, 8, 128, 32, k.cuda(), v.cuda(), OS.n_selected(64, 16, 0.2), 0.5)
    kb = torch.zeros((2, 8, 32, 128), dtype=torch.bfloat16, device="cuda")
    mask = torch.ones((2, 32), dtype=torch.uint8, device="cuda")
    layer.step(qp.cuda(), kb, kb, mask, True)
    layer.step(q.cuda(), kb, kb, mask, False)
    torch.cuda.synchronize()
    want = OL.token_mse(f64(q), f64(qp))
    assert np.array_equal(layer.mse.cpu().numpy(), want)
    assert np.array_equal(layer.active.cpu().numpy().astype(bool), want > np.float32(0.5))
    assert fb.fb_device_error() == 0


W_SMALL = W.get("sparse64k").with_(n_prefix=3000, h_q=8, h_kv=2, block=8, steps=6)


@pytest.mark.parametrize("delta", [0.01, 1e30, -1.0])
def test_losa_schedule_small(fb, delta):
    stats = run(fb, W_SMALL, 5, delta)
    if delta == 0.01:
        assert any(0 < a < W_SMALL.block for a, _ in stats), "want steps with active and stable tokens"


def test_losa_schedule_full_size(fb):
    """sparse64k shapes (N = 65536, 4096 pages, 820 selected, 32 / 8 heads, B = 4):
    the union over active rows only is smaller than over all rows."""
    w = W.get("sparse64k")
    stats = run(fb, w, 6, 0.01, steps=8)
    dens = [np.mean([bin(int(x)).count("1") for x in u.reshape(-1)]) / 32 for a, u in stats if a > 0]
    assert dens and max(dens) < 0.8
