"""The FMA-pipe base-2 exponential of the tcgen05 pass (exp2_fma in fb_ptx.cuh).

CPU: the cubic's coefficients in the kernel source are the minimax fit that
gen_exp2_poly.py derives (relative error on [-1/2, 1/2], p(0) = 1), and in float64
they stay within the stated bound.  GPU: the device function, through
fb_exp2_fma, against float64 2^x and against CUDA's exp2f (torch.exp2 in float32)
over the whole input range the softmax feeds it, with the stated bound; exact at
integers; 0 below -125 and at -inf.
"""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_diffusion_attention_prefix_b200", "csrc")
BOUND = 1.02e-4  # the fit's 1.013e-4 plus float32 evaluation


def kernel_coefficients():
    src = open(os.path.join(CSRC, "fb_ptx.cuh")).read()
    body = src[src.index("float exp2_fma(float x)"):]
    body = body[:body.index("\n}\n")]
    line = [ln for ln in body.splitlines() if "const float p = " in ln][0]
    lits = [float(v) for v in re.findall(r"(\d+\.\d+(?:e-?\d+)?)f", line)]
    c3, c2, c1, c0 = lits  # Horner order in the source
    return np.array([c0, c1, c2, c3])


def test_coefficients_are_the_refit():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", os.path.join(CSRC, "gen_exp2_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    coef, err = gen.fit()
    got = kernel_coefficients()
    assert got[0] == 1.0
    np.testing.assert_allclose(got, coef, rtol=1e-12, atol=0)
    assert err <= 1.0130e-4
    f = np.linspace(-0.5, 0.5, 100001)
    rel = np.abs(np.polyval(got[::-1], f) / np.exp2(f) - 1.0)
    assert rel.max() <= 1.0130e-4
    # minimax: the error equioscillates, so it touches its bound at both ends
    assert rel[0] > 0.9 * rel.max() and rel[-1] > 0.9 * rel.max()


def test_range_reduction_in_float32_numpy():
    # the same steps in float32 on the CPU: round by the 1.5 * 2^23 shift, cubic, exponent add
    c = kernel_coefficients().astype(np.float32)
    x = np.concatenate([np.linspace(-125, 8, 400001, dtype=np.float32), np.arange(-125, 9, dtype=np.float32)])
    big = np.float32(12582912.0)
    t = (x + big).astype(np.float32)
    f = (x - (t - big)).astype(np.float32)
    assert np.abs(f).max() <= 0.5
    p = (((c[3] * f + c[2]) * f + c[1]) * f + c[0]).astype(np.float32)
    r = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).view(np.float32)
    rel = np.abs(r.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= BOUND


@pytest.mark.gpu
def test_device_exp2_fma_error_bound(fb):
    import torch
    x = np.concatenate([
        np.linspace(-125.0, 8.0, 2_000_001),
        np.random.default_rng(3).uniform(-125.0, 8.0, 1_000_000),
        np.arange(-125, 9) + 0.5, np.arange(-125, 9) - 0.5,   # rounding ties: f = +-1/2
        np.arange(-125, 9, dtype=np.float64),
    ]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    y = fb.fb_exp2_fma(xd)
    ref_f32 = torch.exp2(xd)  # CUDA's exp2f
    torch.cuda.synchronize()
    yy = y.cpu().numpy().astype(np.float64)
    truth = np.exp2(x.astype(np.float64))
    inr = x >= -125.0
    assert np.all(yy[~inr] == 0.0)
    rel = np.abs(yy[inr] / truth[inr] - 1.0)
    assert rel.max() <= BOUND, f"max relative error {rel.max():.3e}"
    rel_f = np.abs(yy[inr] / ref_f32.cpu().numpy().astype(np.float64)[inr] - 1.0)
    assert rel_f.max() <= BOUND + 2.0 ** -21, f"vs exp2f: {rel_f.max():.3e}"
    ints = np.arange(-125, 9)
    yi = fb.fb_exp2_fma(torch.from_numpy(ints.astype(np.float32)).cuda()).cpu().numpy()
    assert np.array_equal(yi.astype(np.float64), np.exp2(ints.astype(np.float64)))


@pytest.mark.gpu
def test_device_exp2_fma_underflow_and_inf(fb):
    import torch
    x = torch.tensor([-125.5, -126.0, -130.0, -1e30, float("-inf"), -125.0], device="cuda")
    y = fb.fb_exp2_fma(x).cpu().numpy()
    assert np.array_equal(y[:5], np.zeros(5, np.float32))
    assert y[5] == np.float32(2.0 ** -125)
    e = torch.empty((0,), device="cuda")
    assert fb.fb_exp2_fma(e).numel() == 0
