"""Per-head similarity estimate for the gamma gate (float64).

Test infrastructure only (see :mod:`oracle`).

FlashBlock technical summary (gist.science, paper 2602.05305), "Adaptive reuse
strategies", per-head selection: in the video setting the method estimates, for
each head, how similar the current denoising step is to the cached one, and only
heads whose estimated similarity is above gamma reuse their cache.  The pages do
not give the estimator.

Readings where the pages are silent:
  S1  the similarity of head h is the cosine between its block queries now (Q_h,
      B x D, flattened) and the queries its cached A_out was computed with (its
      queries at its last recompute): a cached row is stale exactly as far as its
      query has moved.
  S2  the sums run in one plain order, so that every implementation produces the
      same bits and the gate decision (sim > gamma, in float32) is reproducible:
      each row's products are summed in ascending d, starting from 0 (float64;
      the products of float32 or bfloat16 inputs are exact in float64, so every
      term costs one rounding), which gives the row's dot product; the row dot
      products are then added one after another in ascending row order, starting
      from 0.  Three such sums are formed: <Q, R>, <Q, Q>, <R, R>.
  S3  sim = <Q, R> / sqrt(<Q, Q> <R, R>) in float64, then rounded to float32; a
      zero norm gives sim = 0 (no evidence of similarity: recompute).
  S4  after a step, the reference queries of the heads that recomputed become
      their current queries; heads that reused keep theirs.
"""
from __future__ import annotations

import numpy as np


def _ordered_sum(row_terms: np.ndarray) -> float:
    """Sum of the per-row values [B] in the order of reading S2: one after another,
    in ascending row order, starting from 0."""
    total = 0.0
    for x in np.asarray(row_terms, np.float64).tolist():
        total = total + x
    return float(total)


def _row_dots(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Per-row sum over d of a[:, d] * b[:, d], in ascending d (float64)."""
    acc = np.zeros(a.shape[0])
    for d in range(a.shape[1]):
        acc = acc + a[:, d] * b[:, d]
    return acc


def head_similarity(q: np.ndarray, q_ref: np.ndarray) -> np.ndarray:
    """float32 [b, H_q]: reading S1-S3 for every (batch element, head)."""
    q = np.asarray(q, np.float64)
    r = np.asarray(q_ref, np.float64)
    b, hq = q.shape[:2]
    out = np.zeros((b, hq), dtype=np.float32)
    for bi in range(b):
        for h in range(hq):
            dqr = _ordered_sum(_row_dots(q[bi, h], r[bi, h]))
            dqq = _ordered_sum(_row_dots(q[bi, h], q[bi, h]))
            drr = _ordered_sum(_row_dots(r[bi, h], r[bi, h]))
            den = np.sqrt(dqq * drr)
            out[bi, h] = np.float32(dqr / den) if den > 0.0 else np.float32(0.0)
    return out


def refresh_reference(q: np.ndarray, q_ref: np.ndarray, reuse: np.ndarray) -> np.ndarray:
    """Reading S4: the reference queries after a step."""
    out = np.array(q_ref, copy=True)
    rec = ~np.asarray(reuse, bool)
    out[rec] = np.asarray(q)[rec]
    return out
