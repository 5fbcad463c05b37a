"""The FlashBlock cached step: gates, prefix cache and in-block merge (float64).

Test infrastructure only (see :mod:`oracle`).

Follows the FlashBlock technical summary (gist.science, paper 2602.05305):

* "1. Problem definition": block diffusion denoises a block of B tokens over
  several steps; each step attends from the block's queries to the prefix KV
  cache and to the block itself.
* "2. Methodology / Core mechanism": J_in = the current block's tokens,
  J_out = the tokens outside it (the prefix cache).  (A_out, L_out) is computed
  over J_out, cached, and reused by later steps; each step computes (A_in, L_in)
  and recombines with the merge equation (:func:`oracle.attention.merge`).
* "Adaptive reuse strategies":
  - threshold reuse: with M^{s+1} the number of updated tokens, the cache is
    reused if M^{s+1} < tau, and recomputed otherwise;
  - per-head selection (video): only heads whose estimated similarity is above
    gamma reuse the cache.

Readings where the pages are silent:
  R3  tau: strict ``M < tau`` reuses; ``M >= tau`` recomputes.
  R4  gamma: strict ``sim > gamma`` reuses (compared in float32, as given).
  R5  tau is one decision per batch element; gamma one per (batch, head).
  R6  step 0 of a block always recomputes (there is no cache yet; the LoSA
      page likewise runs the first step of a block densely).
  R7  the cache holds the result of the last recompute; a reuse step leaves it
      untouched, even for rows whose query changed since.
  R8  J_in is all B block tokens, attended bidirectionally; J_out is the whole prefix.
  R9  the similarity is an input (the pages give no estimator).
  R10 with both gates, a head reuses iff both say reuse.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

from .attention import attend, merge


def updated_count(mask: np.ndarray) -> np.ndarray:
    """M^{s+1} per batch element: the number of block tokens marked updated (a
    nonzero mask entry marks a token, whatever its value)."""
    m = np.asarray(mask)
    return (m != 0).reshape(m.shape[0], -1).sum(axis=1).astype(np.int64)


def tau_reuse(M: np.ndarray, tau: int, first_step: bool) -> np.ndarray:
    """Threshold gate: reuse iff this is not the block's first step and M < tau."""
    if first_step:
        return np.zeros(M.shape, dtype=bool)
    return M < tau


def gamma_reuse(sim: Optional[np.ndarray], gamma: float, first_step: bool, shape) -> np.ndarray:
    """Per-head gate: reuse iff not the first step and sim > gamma (float32 compare).

    ``sim is None`` means no per-head gate: every head passes it.
    """
    if first_step:
        return np.zeros(shape, dtype=bool)
    if sim is None:
        return np.ones(shape, dtype=bool)
    return np.asarray(sim, dtype=np.float32) > np.float32(gamma)


def decisions(mask, first_step: bool, tau: int, sim, gamma: float, h_q: int):
    """(M [b], reuse [b, H_q]) for one step: reuse = tau-reuse AND gamma-reuse."""
    M = updated_count(mask)
    t = tau_reuse(M, tau, first_step)                       # [b]
    g = gamma_reuse(sim, gamma, first_step, (M.shape[0], h_q))
    return M, (t[:, None] & g)


def prefix_attention_rows(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """(A_out, L_out) of query rows [R, D] over one KV head's prefix k/v [N, D]."""
    return attend(q_rows, k, v, scale)


def prefix_attention(q, k_cache, v_cache, scale):
    """(A_out, L_out) [b, H_q, B, D] / [b, H_q, B] over J_out = the whole prefix.

    Query head h reads KV head g = h // (H_q / H_kv) (grouped-query layout).
    """
    b, hq, B, D = q.shape
    hk = k_cache.shape[1]
    G = hq // hk
    A = np.zeros((b, hq, B, v_cache.shape[-1]))
    L = np.zeros((b, hq, B))
    for bi in range(b):
        for h in range(hq):
            A[bi, h], L[bi, h] = attend(q[bi, h], k_cache[bi, h // G], v_cache[bi, h // G], scale)
    return A, L


def block_attention(q, k_blk, v_blk, scale):
    """(A_in, L_in) over J_in = the B tokens of the current block (bidirectional)."""
    return prefix_attention(q, k_blk, v_blk, scale)


def dense_attention(q, k_cache, v_cache, k_blk, v_blk, scale):
    """Standard block-diffusion attention: one softmax over J_out U J_in together.

    This is what every step computes without caching; it is the plain definition
    the merge reproduces exactly when the cache is fresh.
    """
    k_all = np.concatenate([k_cache, k_blk], axis=2)
    v_all = np.concatenate([v_cache, v_blk], axis=2)
    return prefix_attention(q, k_all, v_all, scale)


@dataclasses.dataclass
class StepResult:
    M: np.ndarray          # int64 [b]
    reuse: np.ndarray      # bool [b, H_q]
    a_full: np.ndarray     # [b, H_q, B, D]
    l_full: np.ndarray     # [b, H_q, B]
    a_out: np.ndarray      # cache after the step
    l_out: np.ndarray


class CachedBlockAttention:
    """Stateful oracle of one attention layer over one block's denoising steps."""

    def __init__(self, k_cache, v_cache, h_q: int, scale: float):
        self.k = np.asarray(k_cache, dtype=np.float64)
        self.v = np.asarray(v_cache, dtype=np.float64)
        self.h_q = h_q
        self.scale = scale
        self.a_out: Optional[np.ndarray] = None
        self.l_out: Optional[np.ndarray] = None

    def step(self, q, k_blk, v_blk, mask, first_step: bool, tau: int,
             sim=None, gamma: float = 0.0) -> StepResult:
        q = np.asarray(q, dtype=np.float64)
        b, hq, B, D = q.shape
        G = hq // self.k.shape[1]
        M, reuse = decisions(np.asarray(mask), first_step, tau, sim, gamma, hq)
        if self.a_out is None:
            if not first_step:
                raise ValueError("the first step of a block must have first_step=True")
            self.a_out = np.zeros((b, hq, B, self.v.shape[-1]))
            self.l_out = np.full((b, hq, B), -np.inf)
        for bi in range(b):
            for h in range(hq):
                if not reuse[bi, h]:           # recompute: refresh the cached rows
                    self.a_out[bi, h], self.l_out[bi, h] = attend(
                        q[bi, h], self.k[bi, h // G], self.v[bi, h // G], self.scale)
        a_in, l_in = block_attention(q, np.asarray(k_blk, np.float64),
                                     np.asarray(v_blk, np.float64), self.scale)
        a_full, l_full = merge(self.a_out, self.l_out, a_in, l_in)
        return StepResult(M=M, reuse=reuse, a_full=a_full, l_full=l_full,
                          a_out=self.a_out.copy(), l_out=self.l_out.copy())

    def finish_block(self, k_blk, v_blk) -> None:
        """Block transition (:mod:`oracle.transition`): the block's K/V join the
        prefix; the next block starts afresh (first step recomputes)."""
        from .transition import append_block
        self.k, self.v = append_block(self.k, self.v, k_blk, v_blk)
        self.a_out = None
        self.l_out = None
