"""Softmax attention over a key set, carried as (A, L), and the log-space merge.

Test infrastructure only (see :mod:`oracle`).

FlashBlock technical summary, "2. Methodology / Core mechanism": the full
attention output of a query is split into a part over the tokens of the current
block (J_in) and a part over the tokens outside it (J_out).  Each part is kept
as its normalised output A and its log-normaliser L = log Z, and the two are
recombined in log space:

    m      = max(L_out, L_in)
    A_full = (e^{L_out - m} A_out + e^{L_in - m} A_in) / (e^{L_out - m} + e^{L_in - m})

For a key set J and query q (score s_j = scale * q . k_j):
    Z_J = sum_{j in J} e^{s_j},   L_J = ln Z_J,   A_J = sum_{j in J} (e^{s_j} / Z_J) v_j.
The pages write "log" without a base; natural log is used (reading R2).  An empty
key set has Z = 0: L = -inf and A = 0 (the identity of the merge).

The merge also returns L_full = m + ln(e^{L_out - m} + e^{L_in - m}) = ln(Z_out + Z_in),
the log-normaliser of the union, so that merges compose.

All arithmetic is float64.  Inputs in bf16/fp32 are widened exactly by the caller.
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """(A, L) of each query row of ``q`` [R, D] over the keys ``k``/``v`` [n, D].

    Plain definition: s = scale * q k^T; L = ln sum_j e^{s_j} computed as
    max + ln sum e^{s - max}; A = sum_j e^{s_j - L} v_j.  n == 0 gives (0, -inf).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    R, D = q.shape
    if k.shape[0] == 0:
        return np.zeros((R, v.shape[1])), np.full(R, NEG_INF)
    s = scale * (q @ k.T)                      # [R, n]
    m = s.max(axis=1)
    e = np.exp(s - m[:, None])
    z = e.sum(axis=1)
    L = m + np.log(z)
    A = (e @ v) / z[:, None]
    return A, L


def attend_masked(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, keep: np.ndarray):
    """Like :func:`attend`, but each row r attends only to the keys j with keep[r, j].

    Rows with no kept key get (0, -inf).
    """
    q = np.asarray(q, dtype=np.float64)
    R = q.shape[0]
    A = np.zeros((R, v.shape[1]))
    L = np.full(R, NEG_INF)
    for r in range(R):
        idx = np.nonzero(keep[r])[0]
        if idx.size:
            a, l = attend(q[r:r + 1], k[idx], v[idx], scale)
            A[r], L[r] = a[0], l[0]
    return A, L


def merge(a1: np.ndarray, l1: np.ndarray, a2: np.ndarray, l2: np.ndarray):
    """The FlashBlock log-space merge of two partial results (A1, L1) and (A2, L2).

    Follows the merge equation term by term: m = max(L1, L2), w_k = e^{L_k - m},
    A = (w1 A1 + w2 A2) / (w1 + w2), and L = m + ln(w1 + w2).  Where both L are
    -inf (two empty key sets) the result is the empty result (0, -inf).
    ``a*`` are [..., D], ``l*`` are [...].
    """
    a1 = np.asarray(a1, dtype=np.float64)
    a2 = np.asarray(a2, dtype=np.float64)
    l1 = np.asarray(l1, dtype=np.float64)
    l2 = np.asarray(l2, dtype=np.float64)
    m = np.maximum(l1, l2)
    both_empty = np.isneginf(m)
    m_safe = np.where(both_empty, 0.0, m)
    w1 = np.where(np.isneginf(l1), 0.0, np.exp(l1 - m_safe))
    w2 = np.where(np.isneginf(l2), 0.0, np.exp(l2 - m_safe))
    den = w1 + w2
    den_safe = np.where(both_empty, 1.0, den)
    A = (w1[..., None] * a1 + w2[..., None] * a2) / den_safe[..., None]
    A = np.where(both_empty[..., None], 0.0, A)
    L = np.where(both_empty, NEG_INF, m_safe + np.log(den_safe))
    return A, L


def merge_all(parts):
    """Fold :func:`merge` over a list of (A, L) partials, left to right."""
    A, L = parts[0]
    for a, l in parts[1:]:
        A, L = merge(A, L, a, l)
    return A, L
