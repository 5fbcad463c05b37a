"""GPU parity of the per-head similarity estimate (fb_head_similarity) and the
reference refresh against the CPU oracle (oracle.similarity).

The estimate decides an integer (the gamma gate), so it is compared bit for bit:
both sides sum in the same fixed order in float64 and round once to float32.
"""
import math

import numpy as np
import pytest
import torch

from block_diffusion_attention_prefix_b200 import workloads as W
from oracle import flashblock as OF
from oracle import similarity as OSim

pytestmark = pytest.mark.gpu


def f64(t):
    return t.detach().to("cpu").double().numpy()


def sim_ws(fb, sh):
    n = fb.fb_similarity_workspace_bytes(sh)
    return torch.zeros(((n + 15) // 16 * 16,), device="cuda", dtype=torch.uint8)


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("bf16", 64), ("f32", 64), ("f32", 96)])
@pytest.mark.parametrize("B", [1, 4, 255, 256, 257, 700])
def test_similarity_bit_exact(fb, dtype, D, B):
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    g = torch.Generator().manual_seed(B * 10 + D)
    b, hq, hkv = 2, 4, 2
    q = torch.randn((b, hq, B, D), generator=g).to(td)
    r = torch.randn((b, hq, B, D), generator=g).to(td)
    r[0, 1] = q[0, 1]                    # identical
    r[1, 2] = (-2.0 * q[1, 2].float()).to(td)  # negated and scaled
    r[1, 3] = 0                          # zero norm
    mix = torch.rand((B, 1), generator=g) < 0.3
    r[0, 3] = torch.where(mix, r[0, 3], q[0, 3])  # 70 % of the rows unchanged
    sh = fb.make_shape(b, hq, hkv, D, B, 0, dtype)
    sim = torch.full((b, hq), 7.0, device="cuda")
    fb.fb_head_similarity(sh, q.cuda(), r.cuda(), sim, sim_ws(fb, sh))
    torch.cuda.synchronize()
    want = OSim.head_similarity(f64(q), f64(r))
    assert np.array_equal(sim.cpu().numpy(), want), (sim.cpu().numpy(), want)
    assert fb.fb_device_error() == 0


def test_similarity_video_block_size(fb):
    # the video layer's block: 4680 queries per head, 12 heads, D = 128
    g = torch.Generator().manual_seed(5)
    q = torch.randn((1, 12, 4680, 128), generator=g).to(torch.bfloat16)
    r = (q.float() + 0.3 * torch.randn(q.shape, generator=g)).to(torch.bfloat16)
    sh = fb.make_shape(1, 12, 12, 128, 4680, 0, "bf16")
    sim = torch.zeros((1, 12), device="cuda")
    ws = sim_ws(fb, sh)
    for _ in range(2):  # the workspace counters return to zero
        fb.fb_head_similarity(sh, q.cuda(), r.cuda(), sim, ws)
    torch.cuda.synchronize()
    assert np.array_equal(sim.cpu().numpy(), OSim.head_similarity(f64(q), f64(r)))


def test_refresh_reference_copies_recomputed_heads(fb):
    g = torch.Generator().manual_seed(6)
    q = torch.randn((2, 3, 37, 64), generator=g).to(torch.bfloat16)
    r = torch.randn((2, 3, 37, 64), generator=g).to(torch.bfloat16)
    reuse = torch.tensor([[1, 0, 1], [0, 0, 1]], dtype=torch.uint8)
    sh = fb.make_shape(2, 3, 3, 64, 37, 0, "bf16")
    rd = r.cuda()
    fb.fb_refresh_reference(sh, q.cuda(), rd, reuse.cuda())
    torch.cuda.synchronize()
    want = OSim.refresh_reference(f64(q), f64(r), reuse.numpy().astype(bool))
    assert np.array_equal(f64(rd), want)


@pytest.mark.parametrize("B,gamma", [(16, 0.8), (100, 0.75)])
def test_estimated_gamma_schedule(fb, B, gamma):
    """Steps gated by the on-device estimate (tau off): decisions bit-exact, outputs
    within the bf16 tolerance; B = 16 takes the fused step, B = 100 the large-block path."""
    w = W.get("dlm8b_b16").with_(h_q=8, h_kv=2, block=B, n_prefix=1500, tau=B + 1, steps=6)
    seed = 31
    k, v = W.prefix_kv(w, seed)
    layer = fb.CachedAttentionLayer(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, k.cuda(), v.cuda())
    ref = OF.CachedBlockAttention(f64(k), f64(v), w.h_q, 1 / math.sqrt(w.head_dim))
    q_ref = None
    decisions = []
    for s in W.block_schedule(w, seed):
        layer.step_estimated(s.q.cuda(), s.k_blk.cuda(), s.v_blk.cuda(), s.mask.cuda(), s.first, w.tau, gamma)
        q = f64(s.q)
        sim = OSim.head_similarity(q, q_ref) if not s.first else np.zeros((w.batch, w.h_q), np.float32)
        r = ref.step(q, f64(s.k_blk), f64(s.v_blk), s.mask.numpy(), s.first, w.tau, sim, gamma)
        q_ref = OSim.refresh_reference(q, q if q_ref is None else q_ref, r.reuse)
        torch.cuda.synchronize()
        if not s.first:
            assert np.array_equal(layer.sim.cpu().numpy(), sim), f"step {s.index}: sim"
        assert np.array_equal(layer.dec_reuse.cpu().numpy().astype(bool), r.reuse), f"step {s.index}: decisions"
        err = np.abs(f64(layer.a_full) - r.a_full).max()
        assert err <= 2e-2, f"step {s.index}: A_full {err}"
        decisions.append(r.reuse.copy())
    flat = np.stack(decisions[1:])
    assert flat.any() and not flat.all(), "want both reusing and recomputing heads"
    assert fb.fb_device_error() == 0
