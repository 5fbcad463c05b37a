"""LoSA-style per-token reuse with sparse attention for the active tokens (float64).

Test infrastructure only (see :mod:`oracle`).

Follows "LoSA: Locality Aware Sparse Attention for Block-Wise Diffusion Language
Models" (gist.science, paper 2604.12056):
* "1. The problem: KV inflation": with B queries each selecting its own KV
  positions, the memory traffic is set by the union of the selections;
* "2. Methodology": between two denoising steps only a few tokens change much.
  Active tokens (large change of their queries) get sparse attention over the
  prefix (QUEST as the page selector); stable tokens reuse the prefix attention
  of the previous step; the union of KV pages is taken over the active tokens
  only; the first step of a block runs dense attention to initialise; the
  locality score is the MSE between the queries of step t and step t - 1.
The prefix result is then combined with the block's own keys by the FlashBlock
merge (FlashBlock technical summary, "Core mechanism"), as in the cached step.

Readings where the pages are silent:
  L1  the locality score of token i is the mean over all query heads and channels
      of (q_t - q_{t-1})^2, in float64 in a fixed order (per head ascending d, each
      term rounded as a product then a sum; heads in ascending order), divided by
      H_q * D, rounded to float32;
  L2  a token is active iff its score is above the threshold delta (strict, float32);
  L3  every query row (head) of an active token gets sparse attention over its own
      top-k pages (the page-bound selector of the sparse mode, k = ceil(density *
      pages)); that result becomes the row's cached prefix attention;
  L4  rows of stable tokens keep their cached prefix attention (dense from the
      block's first step, or their last sparse result);
  L5  the pages a step streams for a KV group are the union of its active rows'
      selections.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from .attention import attend, attend_masked, merge
from .flashblock import block_attention
from .sparse import (key_mask_from_pages, n_pages, n_selected, page_estimates, page_minmax, select_pages,
                     union_bitmap)


def token_mse(q: np.ndarray, q_prev: np.ndarray) -> np.ndarray:
    """float32 [b, B]: reading L1."""
    q = np.asarray(q, np.float64)
    p = np.asarray(q_prev, np.float64)
    b, hq, B, D = q.shape
    head_sums = np.zeros((b, hq, B))
    for d in range(D):                      # per head, ascending d
        diff = q[..., d] - p[..., d]
        head_sums = head_sums + diff * diff
    total = np.zeros((b, B))
    for h in range(hq):                     # heads in ascending order
        total = total + head_sums[:, h]
    with np.errstate(over="ignore"):  # scores beyond the float32 range round to inf, as a float32 cast does
        return (total / (hq * D)).astype(np.float32)


def active_tokens(mse: np.ndarray, delta: float) -> np.ndarray:
    """bool [b, B]: reading L2, a token is active iff its score is above delta
    (strict, both in float32)."""
    return np.asarray(mse, np.float32) > np.float32(delta)


@dataclasses.dataclass
class LosaStepResult:
    mse: np.ndarray        # float32 [b, B] (zeros on a first step)
    active: np.ndarray     # bool [b, B]
    sel: np.ndarray        # int64 [b, H_q, B, k]; rows of stable tokens are -1
    union: np.ndarray      # uint32 [b, H_kv, words] over active rows
    a_out: np.ndarray      # cached prefix attention after the step
    l_out: np.ndarray
    a_full: np.ndarray
    l_full: np.ndarray


class LosaAttention:
    """Stateful oracle of one layer over one block's steps in LoSA mode."""

    def __init__(self, k_cache, v_cache, h_q: int, scale: float, page: int, density: float):
        self.k = np.asarray(k_cache, dtype=np.float64)
        self.v = np.asarray(v_cache, dtype=np.float64)
        b, hk, N, D = self.k.shape
        self.h_q, self.scale, self.page = h_q, scale, page
        self.N, self.P = N, n_pages(N, page)
        self.k_sel = n_selected(N, page, density)
        self.bounds = [[page_minmax(self.k[bi, g], page) for g in range(hk)] for bi in range(b)]
        self.a_out = None
        self.l_out = None

    def step(self, q, q_prev, k_blk, v_blk, first_step: bool, delta: float) -> LosaStepResult:
        q = np.asarray(q, dtype=np.float64)
        b, hq, B, D = q.shape
        hk = self.k.shape[1]
        G = hq // hk
        sel = np.full((b, hq, B, self.k_sel), -1, dtype=np.int64)
        if first_step:                      # dense prefix attention initialises the cache
            mse = np.zeros((b, B), np.float32)
            active = np.ones((b, B), bool)
            self.a_out = np.zeros((b, hq, B, D))
            self.l_out = np.full((b, hq, B), -np.inf)
            for bi in range(b):
                for h in range(hq):
                    self.a_out[bi, h], self.l_out[bi, h] = attend(q[bi, h], self.k[bi, h // G], self.v[bi, h // G],
                                                                  self.scale)
        else:
            if self.a_out is None:
                raise ValueError("the first step of a block must have first_step=True")
            mse = token_mse(q, q_prev)
            active = active_tokens(mse, delta)
            for bi in range(b):
                rows = np.nonzero(active[bi])[0]
                if rows.size == 0:
                    continue
                for h in range(hq):
                    g = h // G
                    kmin, kmax = self.bounds[bi][g]
                    picks = select_pages(page_estimates(q[bi, h, rows], kmin, kmax), self.k_sel)
                    sel[bi, h, rows] = picks
                    keep = key_mask_from_pages(picks, self.N, self.page)
                    a, l = attend_masked(q[bi, h, rows], self.k[bi, g], self.v[bi, g], self.scale, keep)
                    self.a_out[bi, h, rows] = a
                    self.l_out[bi, h, rows] = l
        union = np.zeros((b, hk, (self.P + 31) // 32), dtype=np.uint32)
        if not first_step:
            for bi in range(b):
                for g in range(hk):
                    s = sel[bi, g * G:(g + 1) * G].reshape(-1)
                    union[bi, g] = union_bitmap(s[s >= 0], self.P)
        a_in, l_in = block_attention(q, np.asarray(k_blk, np.float64), np.asarray(v_blk, np.float64), self.scale)
        a_full, l_full = merge(self.a_out, self.l_out, a_in, l_in)
        return LosaStepResult(mse=mse, active=active, sel=sel, union=union, a_out=self.a_out.copy(),
                              l_out=self.l_out.copy(), a_full=a_full, l_full=l_full)
