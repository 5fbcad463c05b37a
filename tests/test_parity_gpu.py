"""GPU parity: every libfb entry point against the CPU oracle on seeded inputs.

Integer outputs (M^{s+1}, reuse decisions) must match bit for bit.  Floating
outputs must be within max-abs 1e-5 for fp32 workloads and 2e-2 for bf16
workloads (fp32 accumulation), the tolerances the FlashBlock build targets.
Sizes span several key tiles (64 keys for bf16, 32 for fp32), several splits
and ragged tails.  The dLM-like workloads run at full size on every row here;
the long-context and video workloads at full size are in
test_parity_fullsize_gpu.py.
"""
import math

import numpy as np
import pytest
import torch

from block_diffusion_attention_prefix_b200 import workloads as W
from oracle import attention as OA
from oracle import flashblock as OF

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}


def f64(t):
    return t.detach().to("cpu").double().numpy()


def close(got, want, tol, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    both_inf = np.isneginf(got) & np.isneginf(want)
    assert np.array_equal(np.isneginf(got), np.isneginf(want)), f"{what}: -inf pattern differs"
    g = np.where(both_inf, 0.0, got)
    w = np.where(both_inf, 0.0, want)
    err = np.abs(g - w).max() if g.size else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"
    return err


def rand(shape, dtype, scale=1.0, seed=0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(dtype)


def alloc_pass_outputs(b, hq, B, D, dev="cuda"):
    a = torch.full((b, hq, B, D), 7.0, device=dev, dtype=torch.float32)
    l = torch.full((b, hq, B), 7.0, device=dev, dtype=torch.float32)
    return a, l


def workspace(fb, shape):
    n = fb.fb_workspace_bytes(shape)
    return torch.zeros(((n + 15) // 16 * 16,), device="cuda", dtype=torch.uint8)


# --------------------------------------------------------------------------- merge / gate


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_merge_kernel(fb, dtype):
    b, hq, B, D = 2, 3, 5, 64
    sh = fb.make_shape(b, hq, hq, D, B, 0, dtype)
    g = torch.Generator().manual_seed(1)
    a1 = torch.randn((b, hq, B, D), generator=g)
    a2 = torch.randn((b, hq, B, D), generator=g)
    l1 = torch.randn((b, hq, B), generator=g) * 5
    l2 = torch.randn((b, hq, B), generator=g) * 5
    l1[0, 0, 0] = float("-inf")
    l2[0, 0, 1] = float("-inf")
    l1[1, 2, 3] = l2[1, 2, 3] = float("-inf")
    a1[1, 2, 3] = a2[1, 2, 3] = 0
    l2[1, 1, 1] = l1[1, 1, 1] + 80.0
    out = torch.empty((b, hq, B, D), device="cuda", dtype=torch.float32 if dtype == "f32" else torch.bfloat16)
    lf = torch.empty((b, hq, B), device="cuda")
    fb.fb_merge(sh, a1.cuda(), l1.cuda(), a2.cuda(), l2.cuda(), out, lf)
    A, L = OA.merge(f64(a1), f64(l1), f64(a2), f64(l2))
    close(f64(out), A, 1e-5 if dtype == "f32" else 1e-2, "A")
    close(f64(lf), L, 1e-5, "L")


def test_gate_eval_bit_exact(fb):
    b, hq, B = 6, 8, 16
    sh = fb.make_shape(b, hq, 2, 64, B, 10, "bf16")
    g = torch.Generator().manual_seed(3)
    for trial in range(12):
        mask = (torch.rand((b, B), generator=g) < 0.3).to(torch.uint8)
        mask[0] = 0
        mask[1] = 1
        sim = torch.rand((b, hq), generator=g).to(torch.float32)
        gamma = float(sim[2, 3])                       # one head exactly at gamma: strict > fails
        tau = [0, 1, 2, B // 2, B, B + 1][trial % 6]
        first = trial % 5 == 4
        use_sim = trial % 2 == 0
        dM = torch.full((b,), -1, device="cuda", dtype=torch.int32)
        dR = torch.full((b, hq), 9, device="cuda", dtype=torch.uint8)
        gate = fb.make_gate(mask.cuda(), first, tau, sim.cuda() if use_sim else None, gamma)
        fb.fb_gate_eval(sh, gate, dM, dR)
        M, reuse = OF.decisions(mask.numpy(), first, tau, sim.numpy() if use_sim else None, gamma, hq)
        assert np.array_equal(dM.cpu().numpy(), M)
        assert np.array_equal(dR.cpu().numpy().astype(bool), reuse)


# --------------------------------------------------------------------------- prefix pass


def prefix_case(fb, dtype, b, hq, hkv, D, B, N, seed, row_stride=0, cap=None):
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    cap = N if cap is None else cap
    rs = row_stride or D
    q = rand((b, hq, B, D), td, seed=seed)
    kfull = rand((b, hkv, cap, rs), td, 0.7, seed + 1)
    vfull = rand((b, hkv, cap, rs), td, 1.0, seed + 2)
    k, v = kfull[:, :, :N, :D], vfull[:, :, :N, :D]
    sh = fb.make_shape(b, hq, hkv, D, B, N, dtype, kv_row_stride=rs, kv_head_stride=cap * rs)
    a, l = alloc_pass_outputs(b, hq, B, D)
    ws = workspace(fb, sh)
    fb.fb_prefix_attn(sh, q.cuda(), kfull.cuda(), vfull.cuda(), None, a, l, ws)
    torch.cuda.synchronize()
    assert fb.fb_device_error() == 0
    A, L = OF.prefix_attention(f64(q), f64(k), f64(v), 1 / math.sqrt(D))
    tol = TOL[dtype]
    close(f64(a), A, tol, "A_out")
    close(f64(l), L, tol, "L_out")
    return ws


@pytest.mark.parametrize("N", [0, 1, 31, 32, 33, 1024, 1500])
@pytest.mark.parametrize("D,hq,hkv,B", [(64, 2, 1, 4), (32, 4, 2, 3), (128, 2, 2, 5), (96, 6, 2, 7)])
def test_prefix_f32(fb, N, D, hq, hkv, B):
    prefix_case(fb, "f32", 1, hq, hkv, D, B, N, seed=N + D)


@pytest.mark.parametrize("N", [0, 1, 63, 64, 65, 1000, 4097])
@pytest.mark.parametrize("D,hq,hkv,B", [(128, 32, 8, 4), (128, 8, 2, 16), (64, 8, 4, 8), (128, 3, 3, 3),
                                        (64, 4, 2, 37), (128, 8, 2, 8)])
def test_prefix_bf16(fb, N, D, hq, hkv, B):
    prefix_case(fb, "bf16", 1, hq, hkv, D, B, N, seed=N * 7 + D + B)


def test_prefix_bf16_batched_strided(fb):
    # batch 2, row stride 192 (> D) and head stride with spare capacity
    prefix_case(fb, "bf16", 2, 8, 2, 128, 4, 3000, seed=5, row_stride=192, cap=3500)
    prefix_case(fb, "f32", 2, 4, 2, 64, 4, 300, seed=6, row_stride=96, cap=333)


def test_workspace_counters_return_to_zero(fb):
    ws = prefix_case(fb, "bf16", 1, 8, 2, 128, 4, 5000, seed=9)
    assert int(ws[:256].view(torch.int32).abs().sum()) == 0


def test_prefix_gated_rows_untouched(fb):
    # per-head gate: reusing heads keep their cache rows bit for bit
    b, hq, hkv, D, B, N = 2, 8, 2, 128, 4, 2000
    q = rand((b, hq, B, D), torch.bfloat16, seed=11)
    k = rand((b, hkv, N, D), torch.bfloat16, 0.5, 12)
    v = rand((b, hkv, N, D), torch.bfloat16, 1.0, 13)
    sh = fb.make_shape(b, hq, hkv, D, B, N, "bf16")
    sim = torch.rand((b, hq), generator=torch.Generator().manual_seed(4))
    sim[0, :4] = 0.99    # whole KV group 0 of batch 0 reuses: its CTAs exit early
    mask = torch.zeros((b, B), dtype=torch.uint8)
    a0 = torch.randn((b, hq, B, D)).cuda()
    l0 = torch.randn((b, hq, B)).cuda()
    a, l = a0.clone(), l0.clone()
    ws = workspace(fb, sh)
    gate = fb.make_gate(mask.cuda(), False, 1, sim.cuda(), 0.5)
    fb.fb_prefix_attn(sh, q.cuda(), k.cuda(), v.cuda(), gate, a, l, ws)
    torch.cuda.synchronize()
    A, L = OF.prefix_attention(f64(q), f64(k), f64(v), 1 / math.sqrt(D))
    reuse = sim.numpy() > np.float32(0.5)
    for bi in range(b):
        for h in range(hq):
            if reuse[bi, h]:
                assert torch.equal(a[bi, h], a0[bi, h]) and torch.equal(l[bi, h], l0[bi, h])
            else:
                close(f64(a[bi, h]), A[bi, h], 2e-2, "A")
                close(f64(l[bi, h]), L[bi, h], 2e-2, "L")


# --------------------------------------------------------------------------- in-block pass


@pytest.mark.parametrize("dtype,D", [("f32", 64), ("bf16", 128), ("bf16", 64), ("f32", 128)])
@pytest.mark.parametrize("B", [1, 4, 16, 33, 64, 65, 200])
def test_block_attn(fb, dtype, D, B):
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    b, hq, hkv = 1, 4, 2
    q = rand((b, hq, B, D), td, seed=B)
    kb = rand((b, hkv, B, D), td, 0.8, B + 1)
    vb = rand((b, hkv, B, D), td, 1.0, B + 2)
    sh = fb.make_shape(b, hq, hkv, D, B, 0, dtype)
    a, l = alloc_pass_outputs(b, hq, B, D)
    ws = workspace(fb, sh)
    fb.fb_block_attn(sh, q.cuda(), kb.cuda(), vb.cuda(), a, l, ws)
    A, L = OF.block_attention(f64(q), f64(kb), f64(vb), 1 / math.sqrt(D))
    close(f64(a), A, TOL[dtype], "A_in")
    close(f64(l), L, TOL[dtype], "L_in")


@pytest.mark.parametrize("dtype,B", [("f32", 4), ("bf16", 16), ("bf16", 100)])
def test_block_merge_records_decisions(fb, dtype, B):
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    b, hq, hkv, D = 2, 4, 2, 64
    q = rand((b, hq, B, D), td, seed=21)
    kb = rand((b, hkv, B, D), td, 0.8, 22)
    vb = rand((b, hkv, B, D), td, 1.0, 23)
    a_out = torch.randn((b, hq, B, D)).cuda()
    l_out = (torch.randn((b, hq, B)) * 3).cuda()
    l_out[0, 0, 0] = float("-inf")
    a_out[0, 0, 0] = 0
    mask = torch.zeros((b, B), dtype=torch.uint8)
    mask[1, : B // 2 + 1] = 1
    sh = fb.make_shape(b, hq, hkv, D, B, 0, dtype)
    out = torch.empty((b, hq, B, D), device="cuda", dtype=td)
    lf = torch.empty((b, hq, B), device="cuda")
    dM = torch.full((b,), -1, device="cuda", dtype=torch.int32)
    dR = torch.full((b, hq), 9, device="cuda", dtype=torch.uint8)
    ws = workspace(fb, sh)
    gate = fb.make_gate(mask.cuda(), False, max(1, B // 2))
    fb.fb_block_merge(sh, q.cuda(), kb.cuda(), vb.cuda(), gate, a_out, l_out, out, lf, dM, dR, ws)
    Ai, Li = OF.block_attention(f64(q), f64(kb), f64(vb), 1 / math.sqrt(D))
    A, L = OA.merge(f64(a_out), f64(l_out), Ai, Li)
    close(f64(out), A, TOL[dtype], "A_full")
    close(f64(lf), L, TOL[dtype], "L_full")
    M, reuse = OF.decisions(mask.numpy(), False, max(1, B // 2), None, 0.0, hq)
    assert np.array_equal(dM.cpu().numpy(), M)
    assert np.array_equal(dR.cpu().numpy().astype(bool), reuse)


# --------------------------------------------------------------------------- full schedules


def replay_both(fb, w, seed, steps=None, check_rows=None):
    """Run the seeded schedule through fb_step and the oracle; compare every step."""
    k, v = W.prefix_kv(w, seed)
    kd, vd = k.cuda(), v.cuda()
    layer = fb.CachedAttentionLayer(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, kd, vd)
    ref = OF.CachedBlockAttention(f64(k), f64(v), w.h_q, 1 / math.sqrt(w.head_dim))
    tol = TOL[w.dtype]
    out = []
    for s in W.block_schedule(w, seed, steps):
        sim = None if s.sim is None else s.sim.cuda()
        layer.step(s.q.cuda(), s.k_blk.cuda(), s.v_blk.cuda(), s.mask.cuda(), s.first, w.tau, sim,
                   w.gamma or 0.0)
        r = ref.step(f64(s.q), f64(s.k_blk), f64(s.v_blk), s.mask.numpy(), s.first, w.tau,
                     None if s.sim is None else s.sim.numpy(), w.gamma or 0.0)
        torch.cuda.synchronize()
        assert np.array_equal(layer.dec_M.cpu().numpy(), r.M), f"step {s.index}: M"
        assert np.array_equal(layer.dec_reuse.cpu().numpy().astype(bool), r.reuse), f"step {s.index}: reuse"
        close(f64(layer.a_full), r.a_full, tol, f"step {s.index} A_full")
        close(f64(layer.l_full), r.l_full, tol, f"step {s.index} L_full")
        close(f64(layer.a_out), r.a_out, tol, f"step {s.index} A_out")
        close(f64(layer.l_out), r.l_out, tol, f"step {s.index} L_out")
        out.append((s, r, layer.a_full.clone(), layer.a_out.clone(), layer.l_out.clone()))
    assert fb.fb_device_error() == 0
    return out


def test_schedule_tiny_f32(fb):
    res = replay_both(fb, W.get("tiny_f32"), seed=0)
    # step 5 of seed 0 updates no token: the reuse output equals step 4's bit for bit
    s5 = res[5]
    assert int(s5[0].mask.sum()) == 0
    assert torch.equal(res[5][2], res[4][2])
    assert torch.equal(res[5][3], res[4][3])


@pytest.mark.parametrize("name", ["dlm8b_b4", "dlm8b_b16"])
def test_schedule_dlm8b_full_size(fb, name):
    res = replay_both(fb, W.get(name), seed=1)
    kinds = {bool(r.reuse.any()) for _, r, *_ in res}
    assert kinds == {True, False}, "the schedule must mix reuse and recompute steps"
    for (s0, r0, _, ao0, lo0), (s1, r1, _, ao1, lo1) in zip(res, res[1:]):
        if r1.reuse.all():                            # reuse: cache untouched bit for bit
            assert torch.equal(ao1, ao0) and torch.equal(lo1, lo0)


def test_step_is_deterministic(fb):
    w = W.get("dlm8b_b4").with_(n_prefix=20000)
    k, v = W.prefix_kv(w, 3)
    outs = []
    for _ in range(2):
        layer = fb.CachedAttentionLayer(1, 32, 8, 128, 4, k.cuda(), v.cuda())
        for s in W.block_schedule(w, 3, 4):
            layer.step(s.q.cuda(), s.k_blk.cuda(), s.v_blk.cuda(), s.mask.cuda(), s.first, w.tau)
        outs.append((layer.a_full.clone(), layer.a_out.clone(), layer.l_out.clone()))
    for x, y in zip(*outs):
        assert torch.equal(x, y)


# --------------------------------------------------------------------------- fused step


@pytest.mark.parametrize("variant", [
    dict(name="dlm8b_b4", n_prefix=5000, seed=7),
    dict(name="dlm8b_b4", n_prefix=0, seed=8),                          # empty prefix
    dict(name="dlm8b_b4", n_prefix=3001, block=37, tau=10, seed=9),     # heads straddle row tiles
    dict(name="dlm8b_b16", n_prefix=4000, block=64, tau=20, seed=10),   # 256 rows per KV head: 2 row tiles
    dict(name="dlm8b_b4", n_prefix=3000, block=8, tau=3, seed=14),      # 32 rows per KV head
    dict(name="tiny_f32", n_prefix=777, block=33, h_q=4, h_kv=2, tau=9, seed=11),
])
def test_fused_step_schedules(fb, variant):
    v = dict(variant)
    seed = v.pop("seed")
    w = W.get(v.pop("name")).with_(steps=6, **v)
    replay_both(fb, w, seed)


def test_fused_step_gamma_mixed_heads_in_group(fb):
    # per-head gate inside one KV group (G = 4): some heads reuse, others recompute
    w = W.get("video").with_(h_q=8, h_kv=2, block=16, n_prefix=3000, tau=17, steps=5)
    res = replay_both(fb, w, seed=12)
    mixed = [r.reuse[0, :4] for _, r, *_ in res[1:]]
    assert any(m.any() and not m.all() for m in mixed), "want a step where one KV group mixes decisions"


@pytest.mark.parametrize("name,B", [("dlm8b_b4", 4), ("dlm8b_b16", 16), ("tiny_f32", 4)])
def test_fused_step_equals_two_call_path(fb, name, B):
    """fb_step (one launch) gives the same bits as fb_prefix_attn + fb_block_merge."""
    w = W.get(name).with_(n_prefix=2500, steps=4)
    k, v = W.prefix_kv(w, 13)
    kd, vd = k.cuda(), v.cuda()
    sh = fb.make_shape(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, w.n_prefix, w.dtype)
    ws1, ws2 = workspace(fb, sh), workspace(fb, sh)
    mk = lambda: (torch.zeros((1, w.h_q, w.block, w.head_dim), device="cuda"),  # noqa: E731
                  torch.full((1, w.h_q, w.block), float("-inf"), device="cuda"),
                  torch.zeros((1, w.h_q, w.block, w.head_dim), device="cuda", dtype=w.torch_dtype),
                  torch.zeros((1, w.h_q, w.block), device="cuda"),
                  torch.zeros((1,), device="cuda", dtype=torch.int32),
                  torch.zeros((1, w.h_q), device="cuda", dtype=torch.uint8))
    A, Bt = mk(), mk()
    for s in W.block_schedule(w, 13):
        q, kb, vb, m = s.q.cuda(), s.k_blk.cuda(), s.v_blk.cuda(), s.mask.cuda()
        g = fb.make_gate(m, s.first, w.tau)
        fb.fb_step(sh, q, kd, vd, kb, vb, g, *A, ws1)
        fb.fb_prefix_attn(sh, q, kd, vd, g, Bt[0], Bt[1], ws2)
        fb.fb_block_merge(sh, q, kb, vb, g, Bt[0], Bt[1], Bt[2], Bt[3], Bt[4], Bt[5], ws2)
        torch.cuda.synchronize()
        for x, y in zip(A, Bt):
            assert torch.equal(x, y), f"step {s.index}"


# --------------------------------------------------------------------------- tcgen05 pass (> 16 rows per KV head)


@pytest.mark.parametrize("hq,hkv,B,N", [
    (1, 1, 128, 128),      # exactly one row tile and one key tile
    (2, 2, 128, 1000),     # ragged key tail
    (4, 2, 65, 4097),      # R = 130: two row tiles, the second with 2 rows; GQA
    (1, 1, 300, 0),        # empty prefix
    (1, 1, 200, 50),       # fewer keys than one tile
    (8, 2, 40, 2000),      # R = 160: row tiles straddle query heads
    (1, 1, 128, 7296),     # 114 key tiles: the most splits a 128-row tile combines
    (1, 1, 128, 7327),     # same with a ragged tail
    (12, 12, 1600, 700),   # 13 row tiles x 12 heads fill the GPU: one CTA per row tile, no split
])
def test_prefix_tc(fb, hq, hkv, B, N):
    prefix_case(fb, "bf16", 1, hq, hkv, 128, B, N, seed=hq * 100 + B + N)


def test_prefix_tc_batched_strided(fb):
    # batch 2, row stride 192 and head stride with spare capacity, 2 x 128 rows per KV head
    prefix_case(fb, "bf16", 2, 4, 2, 128, 64, 3000, seed=44, row_stride=192, cap=3100)


def test_prefix_tc_gated_heads(fb):
    # per-head gate with 256 rows per head: reusing heads keep their cache rows bit for bit
    b, hq, hkv, D, B, N = 1, 6, 6, 128, 256, 3000
    q = rand((b, hq, B, D), torch.bfloat16, seed=31)
    k = rand((b, hkv, N, D), torch.bfloat16, 0.5, 32)
    v = rand((b, hkv, N, D), torch.bfloat16, 1.0, 33)
    sh = fb.make_shape(b, hq, hkv, D, B, N, "bf16")
    sim = torch.tensor([[0.1, 0.9, 0.2, 0.8, 0.6, 0.3]])
    mask = torch.zeros((b, B), dtype=torch.uint8)
    a0 = torch.randn((b, hq, B, D)).cuda()
    l0 = torch.randn((b, hq, B)).cuda()
    a, l = a0.clone(), l0.clone()
    ws = workspace(fb, sh)
    fb.fb_prefix_attn(sh, q.cuda(), k.cuda(), v.cuda(), fb.make_gate(mask.cuda(), False, 1, sim.cuda(), 0.5), a, l, ws)
    torch.cuda.synchronize()
    assert fb.fb_device_error() == 0
    A, L = OF.prefix_attention(f64(q), f64(k), f64(v), 1 / math.sqrt(D))
    for h in range(hq):
        if float(sim[0, h]) > 0.5:
            assert torch.equal(a[0, h], a0[0, h]) and torch.equal(l[0, h], l0[0, h])
        else:
            close(f64(a[0, h]), A[0, h], 2e-2, f"A h={h}")
            close(f64(l[0, h]), L[0, h], 2e-2, f"L h={h}")
