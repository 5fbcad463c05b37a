"""Pins of oracle.attention against things other than itself (CPU only).

* library routines: torch float64 scaled_dot_product_attention and logsumexp;
* closed forms: one key, equal keys, two keys give a sigmoid weight;
* hand-derived fixtures in tests/golden/ (merge equation, brute-force attention);
* algebra of the FlashBlock merge: union = dense, associativity, commutativity,
  identity element.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as OA

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def num(x):
    if isinstance(x, (int, float)):
        return float(x)
    return float(eval(x.replace("ln", "math.log"), {"math": math, "inf": math.inf}))


def nums(xs):
    return np.array([[num(v) for v in row] if isinstance(row, list) else num(row) for row in xs])


def rand_qkv(rng, R, n, D, dv=None):
    dv = D if dv is None else dv
    return rng.standard_normal((R, D)), rng.standard_normal((n, D)), rng.standard_normal((n, dv))


@pytest.mark.parametrize("R,n,D,scale", [(1, 1, 4, 0.5), (3, 7, 16, 0.25), (8, 300, 64, 0.125),
                                         (5, 33, 128, 1 / math.sqrt(128))])
def test_attend_matches_torch_sdpa_and_logsumexp(R, n, D, scale):
    rng = np.random.default_rng(R * 1000 + n)
    q, k, v = rand_qkv(rng, R, n, D)
    A, L = OA.attend(q, k, v, scale)
    tq, tk, tv = (torch.from_numpy(x)[None, None] for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)[0, 0].numpy()
    lse = torch.logsumexp(scale * torch.from_numpy(q) @ torch.from_numpy(k).T, dim=1).numpy()
    np.testing.assert_allclose(A, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, lse, rtol=0, atol=1e-12)


def test_weights_sum_to_one():
    rng = np.random.default_rng(1)
    q, k, _ = rand_qkv(rng, 6, 257, 32)
    A, _ = OA.attend(q, 3.0 * k, np.ones((257, 3)), 0.7)
    np.testing.assert_allclose(A, 1.0, rtol=0, atol=1e-12)


def test_one_key_is_identity():
    rng = np.random.default_rng(2)
    q, k, v = rand_qkv(rng, 4, 1, 8)
    A, L = OA.attend(q, k, v, 0.3)
    np.testing.assert_array_equal(A, np.repeat(v, 4, axis=0))
    np.testing.assert_allclose(L, 0.3 * (q @ k[0]), rtol=0, atol=1e-14)


@pytest.mark.parametrize("copies", [2, 3])
def test_equal_keys_mean_and_log_count(copies):
    rng = np.random.default_rng(3)
    q, k, v = rand_qkv(rng, 2, 1, 8)
    kk = np.repeat(k, copies, axis=0)
    vv = rng.standard_normal((copies, 8))
    A, L = OA.attend(q, kk, vv, 0.5)
    np.testing.assert_allclose(A, np.repeat(vv.mean(0, keepdims=True), 2, 0), rtol=0, atol=1e-14)
    np.testing.assert_allclose(L, 0.5 * (q @ k[0]) + math.log(copies), rtol=0, atol=1e-14)


@pytest.mark.parametrize("x", [-3.0, -0.5, 0.0, 0.7, 4.0])
def test_two_scores_give_sigmoid_weight(x):
    # scores {0, x}: the weight of the second key is sigma(x), L = ln(1 + e^x)
    q = np.array([[1.0, 0.0]])
    k = np.array([[0.0, 5.0], [x, -2.0]])
    v = np.array([[1.0, 0.0], [0.0, 1.0]])
    A, L = OA.attend(q, k, v, 1.0)
    sig = 1.0 / (1.0 + math.exp(-x))
    np.testing.assert_allclose(A[0], [1 - sig, sig], rtol=0, atol=1e-15)
    np.testing.assert_allclose(L[0], math.log1p(math.exp(x)), rtol=0, atol=1e-15)


def test_empty_key_set_is_merge_identity():
    A, L = OA.attend(np.ones((3, 4)), np.zeros((0, 4)), np.zeros((0, 5)), 1.0)
    assert A.shape == (3, 5) and np.all(A == 0) and np.all(np.isneginf(L))


def test_golden_attention_cases():
    data = json.load(open(os.path.join(GOLDEN, "attention_cases.json")))
    for c in data["cases"]:
        A, L = OA.attend(nums(c["q"]), nums(c["k"]), nums(c["v"]), c["scale"])
        np.testing.assert_allclose(A, nums(c["a"]), rtol=0, atol=1e-14, err_msg=c["name"])
        np.testing.assert_allclose(L, nums(c["l"]), rtol=0, atol=1e-13, err_msg=c["name"])


def test_golden_merge_cases():
    data = json.load(open(os.path.join(GOLDEN, "merge_cases.json")))
    for c in data["cases"]:
        A, L = OA.merge(np.array(c["a_out"]), num(c["l_out"]), np.array(c["a_in"]), num(c["l_in"]))
        np.testing.assert_allclose(A, c["a_full"], rtol=0, atol=1e-12, err_msg=c["name"])  # 1000+ln3 has ulp 1.1e-13
        want = num(c["l_full"])
        if math.isinf(want):
            assert np.isneginf(L), c["name"]
        else:
            np.testing.assert_allclose(L, want, rtol=0, atol=1e-12, err_msg=c["name"])


@pytest.mark.parametrize("seed", range(6))
def test_merge_of_partition_equals_dense_over_union(seed):
    # the merge over (J_out, J_in) reproduces dense attention over J_out U J_in
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(2, 400))
    q, k, v = rand_qkv(rng, 5, n, 32)
    k *= rng.uniform(0.2, 3.0)
    perm = rng.permutation(n)
    cut = int(rng.integers(1, n))
    J1, J2 = perm[:cut], perm[cut:]
    a1, l1 = OA.attend(q, k[J1], v[J1], 0.2)
    a2, l2 = OA.attend(q, k[J2], v[J2], 0.2)
    A, L = OA.merge(a1, l1, a2, l2)
    Ad, Ld = OA.attend(q, k, v, 0.2)
    np.testing.assert_allclose(A, Ad, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Ld, rtol=0, atol=1e-12)


@pytest.mark.parametrize("parts", [3, 7])
def test_merge_of_many_splits_equals_dense(parts):
    rng = np.random.default_rng(parts)
    q, k, v = rand_qkv(rng, 4, 1000, 16)
    cuts = np.sort(rng.choice(np.arange(1, 1000), parts - 1, replace=False))
    pieces = np.split(np.arange(1000), cuts)
    A, L = OA.merge_all([OA.attend(q, k[p], v[p], 0.5) for p in pieces])
    Ad, Ld = OA.attend(q, k, v, 0.5)
    np.testing.assert_allclose(A, Ad, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Ld, rtol=0, atol=1e-12)


def test_merge_associative_commutative_identity():
    rng = np.random.default_rng(7)
    parts = [(rng.standard_normal((6, 9)), rng.standard_normal(6) * 5) for _ in range(3)]
    (a1, l1), (a2, l2), (a3, l3) = parts
    left = OA.merge(*OA.merge(a1, l1, a2, l2), a3, l3)
    right = OA.merge(a1, l1, *OA.merge(a2, l2, a3, l3))
    np.testing.assert_allclose(left[0], right[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(left[1], right[1], rtol=0, atol=1e-12)
    ab = OA.merge(a1, l1, a2, l2)
    ba = OA.merge(a2, l2, a1, l1)
    np.testing.assert_array_equal(ab[0], ba[0])      # bit-exact: + and max commute
    np.testing.assert_array_equal(ab[1], ba[1])
    ident = OA.merge(a1, l1, np.zeros_like(a1), np.full(6, -np.inf))
    np.testing.assert_array_equal(ident[0], a1)
    np.testing.assert_allclose(ident[1], l1, rtol=0, atol=0)


def test_attend_masked_rows():
    rng = np.random.default_rng(8)
    q, k, v = rand_qkv(rng, 3, 50, 8)
    keep = rng.random((3, 50)) < 0.4
    keep[2] = False
    A, L = OA.attend_masked(q, k, v, 0.4, keep)
    for r in range(2):
        a, l = OA.attend(q[r:r + 1], k[keep[r]], v[keep[r]], 0.4)
        np.testing.assert_array_equal(A[r], a[0])
        np.testing.assert_array_equal(L[r], l[0])
    assert np.all(A[2] == 0) and np.isneginf(L[2])


def test_key_order_does_not_matter():
    # permuting the keys together with their values leaves (A, L) unchanged
    rng = np.random.default_rng(11)
    q, k, v = rand_qkv(rng, 5, 41, 16)
    perm = rng.permutation(41)
    A, L = OA.attend(q, k, v, 0.25)
    Ap, Lp = OA.attend(q, k[perm], v[perm], 0.25)
    np.testing.assert_allclose(Ap, A, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lp, L, rtol=0, atol=1e-12)


def test_common_score_shift_moves_L_only():
    # adding u to every key adds scale * q.u to every score of the row: the weights,
    # hence A, are unchanged and L moves by exactly that amount
    rng = np.random.default_rng(12)
    q, k, v = rand_qkv(rng, 4, 29, 8)
    u = rng.standard_normal(8)
    A, L = OA.attend(q, k, v, 0.5)
    As, Ls = OA.attend(q, k + u, v, 0.5)
    np.testing.assert_allclose(As, A, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Ls, L + 0.5 * (q @ u), rtol=0, atol=1e-12)
