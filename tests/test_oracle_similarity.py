"""Pins of oracle.similarity (CPU only): the per-head similarity estimate.

Pinned by the library (torch float64 cosine similarity of the flattened blocks),
exact summation (math.fsum), and closed forms (identical, negated, scaled and
orthogonal blocks; a zero block)."""
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


def test_pairwise_tree_order_inside_a_chunk():
    # 4 rows: ((a + b) + (c + d)), not ((a + b) + c) + d -- the two differ here
    rows = np.zeros(300)
    rows[:4] = [1.0, 1e-16, -1.0, 1e-16]
    tree = (1.0 + 1e-16) + (-1.0 + 1e-16)
    seq = ((1.0 + 1e-16) + -1.0) + 1e-16
    assert tree != seq
    assert OSim._ordered_sum(rows) == tree


def test_refresh_reference_takes_recomputing_heads():
    q, r = _blocks(3, B=5)
    reuse = np.array([[True, False, True], [False, False, True]])
    out = OSim.refresh_reference(q, r, reuse)
    for bi in range(2):
        for h in range(3):
            np.testing.assert_array_equal(out[bi, h], r[bi, h] if reuse[bi, h] else q[bi, h])
