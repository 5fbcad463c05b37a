"""Sparse attention with a cached residual (FlashBlock x page-level selection), float64.

Test infrastructure only (see :mod:`oracle`).

FlashBlock technical summary (gist.science, paper 2602.05305), "Adaptive reuse
strategies / compatibility with sparse attention": the keys a sparse selector
leaves out are treated as the "out-of-block" set and their residual attention
contribution is cached; the selected keys are attended fresh.  The pages do not
define the selector.  The LoSA page (gist.science, paper 2604.12056, "2.
Methodology") names QUEST as the selector; the page-level bound used here is
the plain reading of a per-page max-score estimate:

  R13  Pages of P consecutive prefix tokens (the last page may be partial and
       uses only its real tokens).  Per page and channel d, kmin_d / kmax_d are
       the min / max of k_d over the page's tokens.  The estimate of page p for a
       query q is  e_p = sum_d max(q_d * kmin_d, q_d * kmax_d), an upper bound of
       q . k over the page.  The softmax scale is left out (ranking only).  Each
       product of two bf16 values is exact in float64 and the sum runs in
       ascending d in float64, so any implementation that sums in the same order
       obtains the same bits.  The top k = ceil(density * n_pages) pages are
       selected per query row, ordered by (estimate descending, page index
       ascending) -- ties go to the lower page index -- and reported as the
       ascending list of page indices.

The stateful algorithm (readings R6, R7 carry over from :mod:`oracle.flashblock`):
  recompute step (first step of the block, or M >= tau):
      estimate pages with the current q, select S per row and freeze it,
      cache the residual (A_res, L_res) = attention over prefix \\ S;
  every step:
      fresh (A_sel, L_sel) over S with the current q,
      A_full = merge(merge(A_sel, A_res), A_in).
"""
from __future__ import annotations

import dataclasses
import math
from fractions import Fraction

import numpy as np

from .attention import attend, attend_masked, merge
from .flashblock import decisions, block_attention


def n_pages(n_prefix: int, page: int) -> int:
    return (n_prefix + page - 1) // page


def n_selected(n_prefix: int, page: int, density) -> int:
    """k = ceil(density * n_pages), at least 1 when there is a page, at most n_pages.

    ``density`` is read as the exact decimal it is written as (0.2 means 1/5), so
    k = ceil(0.2 * 4096) = 820.
    """
    P = n_pages(n_prefix, page)
    k = math.ceil(Fraction(str(density)) * P)
    return min(P, max(1 if P else 0, k))


def page_minmax(k: np.ndarray, page: int):
    """Channel-wise (kmin, kmax) [n_pages, D] of one KV head's keys k [N, D]."""
    N, D = k.shape
    P = n_pages(N, page)
    kmin = np.zeros((P, D))
    kmax = np.zeros((P, D))
    for p in range(P):
        blk = k[p * page:min(N, (p + 1) * page)]
        kmin[p] = blk.min(axis=0)
        kmax[p] = blk.max(axis=0)
    return kmin, kmax


def page_estimates(q_rows: np.ndarray, kmin: np.ndarray, kmax: np.ndarray) -> np.ndarray:
    """e [R, n_pages]: sum over d, in ascending d, of max(q_d kmin_d, q_d kmax_d)."""
    q_rows = np.asarray(q_rows, dtype=np.float64)
    R, D = q_rows.shape
    est = np.zeros((R, kmin.shape[0]), dtype=np.float64)
    for d in range(D):                       # ordered float64 sum
        qd = q_rows[:, d:d + 1]
        est = est + np.maximum(qd * kmin[None, :, d], qd * kmax[None, :, d])
    return est


def select_pages(est: np.ndarray, k_sel: int) -> np.ndarray:
    """Top ``k_sel`` pages per row by (estimate desc, index asc), as ascending indices."""
    R, P = est.shape
    out = np.zeros((R, k_sel), dtype=np.int64)
    for r in range(R):
        order = sorted(range(P), key=lambda p: (-est[r, p], p))
        out[r] = np.sort(np.array(order[:k_sel], dtype=np.int64))
    return out


def union_bitmap(sel_rows: np.ndarray, n_pages_: int) -> np.ndarray:
    """uint32 words: bit p set iff page p is selected by any of the rows."""
    words = np.zeros((n_pages_ + 31) // 32, dtype=np.uint32)
    for p in np.unique(sel_rows):
        words[p // 32] |= np.uint32(1) << np.uint32(p % 32)
    return words


def key_mask_from_pages(sel_rows: np.ndarray, n_prefix: int, page: int) -> np.ndarray:
    """bool [R, N]: key j is in row r's selected set iff its page is selected."""
    R = sel_rows.shape[0]
    keep = np.zeros((R, n_prefix), dtype=bool)
    for r in range(R):
        for p in sel_rows[r]:
            keep[r, p * page:min(n_prefix, (p + 1) * page)] = True
    return keep


@dataclasses.dataclass
class SparseStepResult:
    M: np.ndarray
    reuse: np.ndarray        # bool [b, H_q]
    sel: np.ndarray          # int64 [b, H_q, B, k] frozen selection after the step
    union: np.ndarray        # uint32 [b, H_kv, words]
    a_full: np.ndarray
    l_full: np.ndarray
    a_res: np.ndarray
    l_res: np.ndarray
    a_sel: np.ndarray
    l_sel: np.ndarray


class SparseResidualAttention:
    """Stateful oracle: page-sparse fresh attention plus a cached residual."""

    def __init__(self, k_cache, v_cache, h_q: int, scale: float, page: int, density: float):
        self.k = np.asarray(k_cache, dtype=np.float64)
        self.v = np.asarray(v_cache, dtype=np.float64)
        b, hk, N, D = self.k.shape
        self.h_q, self.scale, self.page = h_q, scale, page
        self.density = density
        self.N = N
        self.P = n_pages(N, page)
        self.k_sel = n_selected(N, page, density)
        self.bounds = [[page_minmax(self.k[bi, g], page) for g in range(hk)] for bi in range(b)]
        self.sel = None
        self.a_res = None
        self.l_res = None

    def step(self, q, k_blk, v_blk, mask, first_step: bool, tau: int) -> SparseStepResult:
        q = np.asarray(q, dtype=np.float64)
        b, hq, B, D = q.shape
        hk = self.k.shape[1]
        G = hq // hk
        M, reuse = decisions(np.asarray(mask), first_step, tau, None, 0.0, hq)
        if self.sel is None:
            if not first_step:
                raise ValueError("the first step of a block must have first_step=True")
            self.sel = np.zeros((b, hq, B, self.k_sel), dtype=np.int64)
            self.a_res = np.zeros((b, hq, B, self.v.shape[-1]))
            self.l_res = np.full((b, hq, B), -np.inf)
        a_sel = np.zeros((b, hq, B, self.v.shape[-1]))
        l_sel = np.full((b, hq, B), -np.inf)
        for bi in range(b):
            for h in range(hq):
                g = h // G
                if not reuse[bi, h]:
                    kmin, kmax = self.bounds[bi][g]
                    est = page_estimates(q[bi, h], kmin, kmax)
                    self.sel[bi, h] = select_pages(est, self.k_sel)
                    keep = key_mask_from_pages(self.sel[bi, h], self.N, self.page)
                    self.a_res[bi, h], self.l_res[bi, h] = attend_masked(
                        q[bi, h], self.k[bi, g], self.v[bi, g], self.scale, ~keep)
                keep = key_mask_from_pages(self.sel[bi, h], self.N, self.page)
                a_sel[bi, h], l_sel[bi, h] = attend_masked(
                    q[bi, h], self.k[bi, g], self.v[bi, g], self.scale, keep)
        union = np.zeros((b, hk, (self.P + 31) // 32), dtype=np.uint32)
        for bi in range(b):
            for g in range(hk):
                union[bi, g] = union_bitmap(self.sel[bi, g * G:(g + 1) * G].reshape(-1), self.P)
        a_pre, l_pre = merge(a_sel, l_sel, self.a_res, self.l_res)
        a_in, l_in = block_attention(q, np.asarray(k_blk, np.float64), np.asarray(v_blk, np.float64),
                                     self.scale)
        a_full, l_full = merge(a_pre, l_pre, a_in, l_in)
        return SparseStepResult(M=M, reuse=reuse, sel=self.sel.copy(), union=union,
                                a_full=a_full, l_full=l_full, a_res=self.a_res.copy(),
                                l_res=self.l_res.copy(), a_sel=a_sel, l_sel=l_sel)

    def finish_block(self, k_blk, v_blk) -> None:
        """Block transition (:mod:`oracle.transition`, readings T1-T3): the block's
        K/V join the prefix, the page bounds the new rows touch are refreshed, k
        follows the grown page count, and the next block starts afresh."""
        from .transition import append_block, update_page_minmax
        n_old = self.N
        self.k, self.v = append_block(self.k, self.v, k_blk, v_blk)
        b, hk, N, D = self.k.shape
        self.bounds = [[update_page_minmax(*self.bounds[bi][g], self.k[bi, g], n_old, self.page)
                        for g in range(hk)] for bi in range(b)]
        self.N = N
        self.P = n_pages(N, self.page)
        self.k_sel = n_selected(N, self.page, self.density)
        self.sel = None
        self.a_res = None
        self.l_res = None
