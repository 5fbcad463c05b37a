"""fb_prefix_attn_noalloc: the prefix pass for callers that cannot allocate.

Some callers cannot call cudaMalloc where they run attention (fixed memory
budgets whose pools are already carved up, hot paths where allocation is not
allowed), so they cannot hand fb_prefix_attn its workspace.  This entry point
keeps the workspace in a static device array owned by the library.

The tests call it through the C-ABI several times in a row (the array keeps the
previous call's contents between them).  Each result must equal fb_prefix_attn
with a caller-allocated workspace bit for bit -- the same kernel runs with the
same split plan, and the pass is deterministic -- and must match the CPU oracle
within the bf16 tolerance of the parity tests.  Gated calls must leave the rows
of reusing heads untouched.  A shape needing more than the array is rejected up
front; a shape whose fused-step workspace is larger than the array but whose
prefix pass alone fits is accepted.

This file is collected last so that a stop-at-first-failure run has already run
every other test; it passes on its own in a fresh process as well.
"""
import math

import numpy as np
import pytest
import torch

from oracle import flashblock as OF

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
SENTINEL = 3.0


def _inputs(seed, b, hq, hkv, D, B, N):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((b, hq, B, D), generator=g).to(torch.bfloat16)
    k = (0.5 * torch.randn((b, hkv, N, D), generator=g)).to(torch.bfloat16)
    v = torch.randn((b, hkv, N, D), generator=g).to(torch.bfloat16)
    return q, k, v


def _f64(t):
    return t.detach().cpu().double().numpy()


def _both(fb, shape, q, k, v, gate, ws):
    """fb_prefix_attn (caller workspace) and fb_prefix_attn_noalloc on the same inputs,
    outputs pre-filled with a sentinel."""
    b, hq, B, D = q.shape
    outs = []
    for _ in range(2):
        outs.append((torch.full((b, hq, B, D), SENTINEL, device="cuda"),
                     torch.full((b, hq, B), SENTINEL, device="cuda")))
    fb.fb_prefix_attn(shape, q, k, v, gate, outs[0][0], outs[0][1], ws)
    fb.fb_prefix_attn_noalloc(shape, q, k, v, gate, outs[1][0], outs[1][1])
    torch.cuda.synchronize()
    return outs


def _check_rows(got, ref, oracle, recompute, what):
    """Recomputed rows: bit-equal to fb_prefix_attn and within tolerance of the oracle.
    Reused rows: the sentinel, untouched."""
    (a_got, l_got), (a_ref, l_ref), (A, L) = got, ref, oracle
    b, hq = recompute.shape
    for bi in range(b):
        for h in range(hq):
            tag = f"{what} b={bi} h={h}"
            if recompute[bi, h]:
                assert torch.equal(a_got[bi, h], a_ref[bi, h]), f"{tag}: A_out differs from fb_prefix_attn"
                assert torch.equal(l_got[bi, h], l_ref[bi, h]), f"{tag}: L_out differs from fb_prefix_attn"
                err_a = np.abs(_f64(a_got[bi, h]) - A[bi, h]).max()
                err_l = np.abs(_f64(l_got[bi, h]) - L[bi, h]).max()
                assert err_a <= TOL_BF16 and err_l <= TOL_BF16, f"{tag}: vs oracle {err_a:.2e} / {err_l:.2e}"
            else:
                assert bool((a_got[bi, h] == SENTINEL).all()) and bool((l_got[bi, h] == SENTINEL).all()), \
                    f"{tag}: a reusing head's row was written"


def _workspace(fb, shape):
    n = fb.fb_workspace_bytes(shape)
    return torch.zeros(((n + 15) // 16 * 16,), dtype=torch.uint8, device="cuda")


def test_noalloc_matches_workspace_entry_point_and_oracle_on_consecutive_calls(fb):
    b, hq, hkv, D, B, N = 2, 32, 8, 128, 4, 32768
    shape = fb.make_shape(b, hq, hkv, D, B, N, "bf16")
    q1, k, v = _inputs(1, b, hq, hkv, D, B, N)
    q2, _, _ = _inputs(2, b, hq, hkv, D, B, N)
    kd, vd = k.cuda(), v.cuda()
    scale = 1 / math.sqrt(D)
    ws = _workspace(fb, shape)

    # mask: batch 0 updates no token (reuses with tau = 2), batch 1 updates three (recomputes)
    mask = torch.tensor([[0, 0, 0, 0], [1, 1, 0, 1]], dtype=torch.uint8, device="cuda")
    sim = torch.rand((b, hq), generator=torch.Generator().manual_seed(7))
    calls = [
        ("ungated", q1, None, np.ones((b, hq), dtype=bool)),
        ("first step", q2, fb.make_gate(mask, True, 2), np.ones((b, hq), dtype=bool)),
        ("tau gate", q1, fb.make_gate(mask, False, 2), np.array([[False] * hq, [True] * hq])),
        ("gamma gate", q2, fb.make_gate(mask, False, 9, sim.cuda(), 0.5), (sim <= 0.5).numpy()),
    ]
    for what, q, gate, recompute in calls:
        got, ref = _both(fb, shape, q.cuda(), kd, vd, gate, ws)[::-1]
        A, L = OF.prefix_attention(_f64(q), _f64(k), _f64(v), scale)
        if gate is not None:
            M, reuse = OF.decisions(mask.cpu().numpy(), bool(gate.first_step), gate.tau,
                                    None if what != "gamma gate" else sim.numpy(), gate.gamma, hq)
            assert np.array_equal(~reuse, recompute)
        assert recompute.any()
        _check_rows(got, ref, (A, L), recompute, what)
    assert fb.fb_device_error() == 0


def test_noalloc_accepts_a_shape_whose_step_workspace_exceeds_the_array(fb):
    # 128 query rows per KV head and 160 (b, KV head) units: the prefix pass alone runs
    # one CTA per row tile over all keys (no split scratch), while the fused step's
    # workspace (split partials plus in-block rows) is larger than the 8 MiB array
    b, hq, hkv, D, B, N = 4, 80, 40, 128, 64, 2048
    shape = fb.make_shape(b, hq, hkv, D, B, N, "bf16")
    assert fb.fb_workspace_bytes(shape) > 8 << 20
    q, k, v = _inputs(3, b, hq, hkv, D, B, N)
    ws = _workspace(fb, shape)
    got, ref = _both(fb, shape, q.cuda(), k.cuda(), v.cuda(), None, ws)[::-1]
    A, L = OF.prefix_attention(_f64(q), _f64(k), _f64(v), 1 / math.sqrt(D))
    _check_rows(got, ref, (A, L), np.ones((b, hq), dtype=bool), "large step workspace")
    assert fb.fb_device_error() == 0


def test_noalloc_rejects_shapes_beyond_the_static_array(fb):
    # a dLM-8B-like layer with 64-token blocks (256 query rows per KV head) needs
    # about 9.7 MB of split partials for its prefix pass: more than 8 MiB
    b, hq, hkv, D, B, N = 1, 32, 8, 128, 64, 32768
    shape = fb.make_shape(b, hq, hkv, D, B, N, "bf16")
    assert fb.fb_workspace_bytes(shape) > 8 << 20
    q = torch.zeros((b, hq, B, D), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((b, hkv, N, D), dtype=torch.bfloat16, device="cuda")
    a = torch.zeros((b, hq, B, D), device="cuda")
    l = torch.zeros((b, hq, B), device="cuda")
    with pytest.raises(fb.FBError) as ei:
        fb.fb_prefix_attn_noalloc(shape, q, kv, kv, None, a, l)
    assert ei.value.status == -5
