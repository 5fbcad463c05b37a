"""Pins of oracle.similarity (CPU only): the per-head similarity estimate.

Pinned by the library (torch float64 cosine similarity of the flattened blocks),
exact summation (math.fsum) within the error bound of recursive summation,
hand-derived values that only the stated summation order gives, and closed forms
(identical, negated, scaled and orthogonal blocks; a zero block)."""
import math

import numpy as np
import pytest
import torch

from oracle import similarity as OSim


def _blocks(seed, b=2, hq=3, B=37, D=16):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((b, hq, B, D)), rng.standard_normal((b, hq, B, D))


@pytest.mark.parametrize("B", [1, 37, 256, 300, 700])
def test_matches_library_cosine(B):
    q, r = _blocks(B, B=B)
    got = OSim.head_similarity(q, r)
    want = torch.nn.functional.cosine_similarity(torch.from_numpy(q.reshape(2, 3, -1)),
                                                 torch.from_numpy(r.reshape(2, 3, -1)), dim=-1, eps=0.0).numpy()
    np.testing.assert_allclose(got, want, atol=2e-7)


def test_ordered_sums_equal_exact_sum():
    q, r = _blocks(1, B=613)
    for bi in range(2):
        for h in range(3):
            rows = OSim._row_dots(q[bi, h], r[bi, h])
            exact = math.fsum((q[bi, h] * r[bi, h]).reshape(-1).tolist())
            assert abs(OSim._ordered_sum(rows) - exact) <= 1e-12 * max(1.0, abs(exact))


def test_closed_forms():
    q, _ = _blocks(2, B=50)
    assert np.all(np.abs(OSim.head_similarity(q, q) - 1.0) <= 1e-7)
    assert np.all(np.abs(OSim.head_similarity(q, -q) + 1.0) <= 1e-7)
    assert np.all(np.abs(OSim.head_similarity(q, 3.5 * q) - 1.0) <= 1e-7)
    # orthogonal: the reference block is q with its two halves of d swapped and one negated
    r = np.concatenate([-q[..., 8:], q[..., :8]], axis=-1)
    x = np.concatenate([q[..., :8], q[..., 8:]], axis=-1)
    y = np.concatenate([x[..., 8:], -x[..., :8]], axis=-1)
    assert np.all(np.abs(OSim.head_similarity(x, y)) <= 1e-7)
    assert np.all(OSim.head_similarity(q, np.zeros_like(q)) == 0.0)


def test_rows_added_in_ascending_order():
    # one channel, four rows whose products are 1, 1e-16, -1, 1e-16.  Added one
    # after another from 0: 1 + 1e-16 rounds to 1, minus 1 gives 0, plus 1e-16
    # gives 1e-16.  (The exact sum is 2e-16; a pairwise tree gives 2^-53, the
    # reverse order 2^-52.)  <Q,Q> = 2 and <R,R> = 4 exactly, so
    # sim = 1e-16 / sqrt(8) rounded to float32.
    q = np.array([1.0, 1e-16, -1.0, 1e-16]).reshape(1, 1, 4, 1)
    r = np.ones_like(q)
    assert OSim.head_similarity(q, r)[0, 0] == np.float32(1e-16 / math.sqrt(8.0))


def test_channels_added_in_ascending_order():
    # the same four products along d of one row: ascending d gives 1e-16 again
    q = np.array([1.0, 1e-16, -1.0, 1e-16]).reshape(1, 1, 1, 4)
    r = np.ones_like(q)
    assert OSim.head_similarity(q, r)[0, 0] == np.float32(1e-16 / math.sqrt(8.0))


def test_sum_error_within_the_sequential_bound():
    # recursive summation of n terms: |error| <= (n - 1) u sum|x_i| (u = 2^-53),
    # against the exact sum (math.fsum is correctly rounded)
    rng = np.random.default_rng(5)
    x = rng.standard_normal(5000) * np.exp(rng.uniform(-20, 20, 5000))
    exact = math.fsum(x.tolist())
    bound = (len(x) - 1) * 2.0 ** -53 * np.abs(x).sum()
    assert abs(OSim._ordered_sum(x) - exact) <= bound


def test_refresh_reference_takes_recomputing_heads():
    q, r = _blocks(3, B=5)
    reuse = np.array([[True, False, True], [False, False, True]])
    out = OSim.refresh_reference(q, r, reuse)
    for bi in range(2):
        for h in range(3):
            np.testing.assert_array_equal(out[bi, h], r[bi, h] if reuse[bi, h] else q[bi, h])
