"""fb_prefix_attn_noalloc: the prefix pass for callers that cannot allocate.

Some callers cannot call cudaMalloc where they run attention (fixed memory
budgets whose pools are already carved up, hot paths where allocation is not
allowed), so they cannot hand fb_prefix_attn its workspace.  This entry point
keeps the workspace in a static device array owned by the library.  The test
calls it through the C-ABI twice in a row (the array keeps the previous call's
contents between them) and checks each result against fb_prefix_attn with a
caller-allocated workspace, within the bf16 tolerance used by the parity tests.
It also checks that a shape needing more than the array is rejected up front.
This file is collected last so that a stop-at-first-failure run has already run
every other test; it passes on its own in a fresh process as well.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


def _inputs(seed, b, hq, hkv, D, B, N):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((b, hq, B, D), generator=g).to(torch.bfloat16).cuda()
    k = (0.5 * torch.randn((b, hkv, N, D), generator=g)).to(torch.bfloat16).cuda()
    v = torch.randn((b, hkv, N, D), generator=g).to(torch.bfloat16).cuda()
    return q, k, v


def test_noalloc_matches_workspace_entry_point_on_two_calls(fb):
    b, hq, hkv, D, B, N = 1, 32, 8, 128, 4, 32768
    shape = fb.make_shape(b, hq, hkv, D, B, N, "bf16")
    q1, k, v = _inputs(1, b, hq, hkv, D, B, N)
    q2, _, _ = _inputs(2, b, hq, hkv, D, B, N)
    mask = torch.ones((b, B), dtype=torch.uint8, device="cuda")
    n = fb.fb_workspace_bytes(shape)
    ws = torch.zeros(((n + 15) // 16 * 16,), dtype=torch.uint8, device="cuda")
    for call, (q, gate) in enumerate([(q1, None), (q2, fb.make_gate(mask, True, 2))]):
        a_ref = torch.zeros((b, hq, B, D), device="cuda")
        l_ref = torch.zeros((b, hq, B), device="cuda")
        a_got = torch.full((b, hq, B, D), 3.0, device="cuda")
        l_got = torch.full((b, hq, B), 3.0, device="cuda")
        fb.fb_prefix_attn(shape, q, k, v, gate, a_ref, l_ref, ws)
        fb.fb_prefix_attn_noalloc(shape, q, k, v, gate, a_got, l_got)
        torch.cuda.synchronize()
        err_a = (a_got - a_ref).abs().max().item()
        err_l = (l_got - l_ref).abs().max().item()
        assert np.isfinite(err_a) and err_a <= TOL_BF16, f"call {call}: A_out differs by {err_a}"
        assert np.isfinite(err_l) and err_l <= TOL_BF16, f"call {call}: L_out differs by {err_l}"
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
