"""GPU parity of the batched fused step: many independent problems in one fb_step.

When the (batch element, KV head, row tile) units of a step fill two waves of the
GPU or more, fb_step writes every reusing row in the reuse-rows kernel (a warp per
row, several CTAs per SM) and runs the prefix pass only on the tiles that
recompute (persistent CTAs for bf16).  These tests replay seeded schedules of
several hundred problems -- some batch elements reusing, others recomputing, at
every step -- and compare every row with the CPU oracle (decisions bit for bit,
floats within the parity tolerance), and check the outputs bit for bit against
the single-wave fused path run on the same problems in slices.
"""
import math

import numpy as np
import pytest
import torch

from oracle import flashblock as OF

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}


def f64(t):
    return t.detach().to("cpu").double().numpy()


def close(got, want, tol, what):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(want)), f"{what}: -inf pattern differs"
    both = np.isneginf(got) & np.isneginf(want)
    err = np.abs(np.where(both, 0.0, got) - np.where(both, 0.0, want)).max()
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


def schedule(b, hq, hkv, D, B, steps, dtype, seed, with_sim=False):
    """Seeded steps: step 0 updates every token; later steps update each token with
    p = 0.25 independently per batch element (fresh q / k / v for updated tokens)."""
    g = torch.Generator().manual_seed(seed)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    q = torch.randn((b, hq, B, D), generator=g)
    kb = torch.randn((b, hkv, B, D), generator=g) * 0.5
    vb = torch.randn((b, hkv, B, D), generator=g)
    out = []
    for s in range(steps):
        mask = torch.ones((b, B), dtype=torch.uint8) if s == 0 else \
            (torch.rand((b, B), generator=g) < 0.25).to(torch.uint8)
        if s > 0:
            upd = mask.bool()
            q = torch.where(upd.view(b, 1, B, 1), torch.randn((b, hq, B, D), generator=g), q)
            kb = torch.where(upd.view(b, 1, B, 1), torch.randn((b, hkv, B, D), generator=g) * 0.5, kb)
            vb = torch.where(upd.view(b, 1, B, 1), torch.randn((b, hkv, B, D), generator=g), vb)
        sim = torch.rand((b, hq), generator=g) if with_sim else None
        out.append((s == 0, q.to(td), kb.to(td), vb.to(td), mask, sim))
    return out


def run_fb(fb, sh, k, v, sched, tau, gamma, dtype, slices=1):
    """fb_step over the schedule; the batch optionally cut into `slices` calls."""
    b, hq, B, D = sched[0][1].shape
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    per = b // slices
    shs = [fb.make_shape(per, sh.h_q, sh.h_kv, D, B, sh.n_prefix, dtype) for _ in range(slices)]
    ws = []
    for s in shs:
        n = fb.fb_workspace_bytes(s)
        ws.append(torch.zeros(((n + 15) // 16 * 16,), device="cuda", dtype=torch.uint8))
    a_out = torch.zeros((b, hq, B, D), device="cuda")
    l_out = torch.full((b, hq, B), float("-inf"), device="cuda")
    res = []
    for first, q, kb, vb, mask, sim in sched:
        a_full = torch.zeros((b, hq, B, D), device="cuda", dtype=td)
        l_full = torch.zeros((b, hq, B), device="cuda")
        dM = torch.full((b,), -1, device="cuda", dtype=torch.int32)
        dR = torch.full((b, hq), 9, device="cuda", dtype=torch.uint8)
        qd, kbd, vbd, md = q.cuda(), kb.cuda(), vb.cuda(), mask.cuda()
        simd = None if sim is None else sim.cuda()
        for i in range(slices):
            sl = slice(i * per, (i + 1) * per)
            gate = fb.make_gate(md[sl].contiguous(), first, tau, None if simd is None else simd[sl].contiguous(),
                                gamma)
            outs = [a_out[sl], l_out[sl], a_full[sl], l_full[sl], dM[sl], dR[sl]]
            if slices > 1:
                outs = [t.clone() for t in outs]
            fb.fb_step(shs[i], qd[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous(), kbd[sl].contiguous(),
                       vbd[sl].contiguous(), gate, *outs, ws[i])
            if slices > 1:
                for dst, src in zip([a_out, l_out, a_full, l_full, dM, dR], outs):
                    dst[sl] = src
        torch.cuda.synchronize()
        res.append(dict(a_full=a_full.cpu(), l_full=l_full.cpu(), a_out=a_out.cpu(), l_out=l_out.cpu(),
                        M=dM.cpu().numpy(), reuse=dR.cpu().numpy().astype(bool)))
    assert fb.fb_device_error() == 0
    return res


@pytest.mark.parametrize("dtype,b,hq,hkv,D,B,N,with_sim", [
    ("bf16", 320, 8, 2, 128, 4, 200, False),    # 640 units of 16 rows: persistent mma.sync pass
    ("bf16", 320, 8, 2, 128, 4, 200, True),     # per-head gate: tiles that mix reusing and recomputing heads
    ("bf16", 160, 8, 2, 128, 16, 130, False),   # 64 rows per KV head (mma.sync 64-row tiles in this mode)
    ("bf16", 300, 4, 4, 64, 8, 77, False),      # D = 64, MHA, 8 rows per head
    ("f32", 1200, 2, 1, 64, 4, 100, False),     # fp32: 1200 units of the CUDA-core pass
])
def test_batched_step_matches_oracle(fb, dtype, b, hq, hkv, D, B, N, with_sim):
    sh = fb.make_shape(b, hq, hkv, D, B, N, dtype)
    g = torch.Generator().manual_seed(b + N)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    k = (torch.randn((b, hkv, N, D), generator=g) * 0.5).to(td)
    v = torch.randn((b, hkv, N, D), generator=g).to(td)
    tau, gamma = (B // 2, 0.5) if not with_sim else (B + 1, 0.5)
    sched = schedule(b, hq, hkv, D, B, 4, dtype, seed=b * 7 + B, with_sim=with_sim)
    got = run_fb(fb, sh, k.cuda(), v.cuda(), sched, tau, gamma, dtype)
    ref = OF.CachedBlockAttention(f64(k), f64(v), hq, 1 / math.sqrt(D))
    mixed = False
    for si, ((first, q, kb, vb, mask, sim), o) in enumerate(zip(sched, got)):
        r = ref.step(f64(q), f64(kb), f64(vb), mask.numpy(), first, tau, None if sim is None else sim.numpy(),
                     gamma)
        assert np.array_equal(o["M"], r.M), f"step {si}: M"
        assert np.array_equal(o["reuse"], r.reuse), f"step {si}: reuse"
        if 0 < r.reuse.sum() < r.reuse.size:
            mixed = True
        for key in ("a_full", "l_full", "a_out", "l_out"):
            close(f64(o[key]), getattr(r, key), TOL[dtype], f"step {si} {key}")
    assert mixed, "want steps where some problems reuse and others recompute"


@pytest.mark.parametrize("dtype,b,hq,hkv,D,B,N,slices", [
    ("bf16", 320, 8, 2, 128, 4, 200, 4),    # 80 problems per slice: 160 units, one split per tile
    ("f32", 1200, 2, 1, 64, 4, 100, 4),     # 300 units per slice
])
def test_batched_step_bit_identical_to_single_wave_path(fb, dtype, b, hq, hkv, D, B, N, slices):
    # Slices small enough for the single-wave plan, whose tiles also run one split each:
    # the same per-tile arithmetic, so the two plans must agree bit for bit.
    sh = fb.make_shape(b, hq, hkv, D, B, N, dtype)
    g = torch.Generator().manual_seed(3)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    k = (torch.randn((b, hkv, N, D), generator=g) * 0.5).to(td).cuda()
    v = torch.randn((b, hkv, N, D), generator=g).to(td).cuda()
    sched = schedule(b, hq, hkv, D, B, 5, dtype, seed=11)
    batched = run_fb(fb, sh, k, v, sched, B // 2, 0.0, dtype)
    sliced = run_fb(fb, sh, k, v, sched, B // 2, 0.0, dtype, slices=slices)
    for si, (x, y) in enumerate(zip(batched, sliced)):
        for key in ("a_full", "l_full", "a_out", "l_out"):
            assert torch.equal(x[key], y[key]), f"step {si} {key}"
        assert np.array_equal(x["M"], y["M"]) and np.array_equal(x["reuse"], y["reuse"])
