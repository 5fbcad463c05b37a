"""Block transition: a finished block joins the prefix (float64).

Test infrastructure only (see :mod:`oracle`).

Follows the FlashBlock technical summary (gist.science, paper 2602.05305),
"1. Problem definition": block diffusion generates a sequence block by block;
each denoising step of the current block attends to the block itself (J_in) and
to the tokens outside it (J_out), which are the earlier blocks.  When a block's
last denoising step is done, its tokens are part of what every later block
attends to as J_out: the prefix grows by one block.

Readings where the pages are silent:
  T1  the keys and values a finished block contributes are its in-block K/V as of
      its last denoising step; they are appended after the prefix, in block order.
  T2  the cached (A_out, L_out) of the finished block is not carried over: the next
      block starts with a first step, which recomputes it (reading R6).
  T3  sparse mode: page bounds depend only on the keys of each page, so after the
      append only the pages the new rows fall in change (the first of them may be
      a partial page that already held prefix rows); the others keep their bounds.
      The number of selected pages follows the grown prefix: k = ceil(density * pages).
"""
from __future__ import annotations

import numpy as np

from .sparse import n_pages


def append_block(k_cache, v_cache, k_blk, v_blk):
    """Prefix K/V [b, H_kv, N, D] with the block's K/V [b, H_kv, B, D] after it."""
    return (np.concatenate([np.asarray(k_cache, np.float64), np.asarray(k_blk, np.float64)], axis=2),
            np.concatenate([np.asarray(v_cache, np.float64), np.asarray(v_blk, np.float64)], axis=2))


def update_page_minmax(kmin, kmax, k_grown, n_old: int, page: int):
    """Page bounds [n_pages, D] of one KV head after its keys grew from n_old rows to
    k_grown [N, D]: pages before the one row n_old falls in are kept, the others
    are taken over their real rows of k_grown (reading T3)."""
    N, D = k_grown.shape
    P = n_pages(N, page)
    first = n_old // page
    new_min = np.zeros((P, D))
    new_max = np.zeros((P, D))
    new_min[:first] = np.asarray(kmin)[:first]
    new_max[:first] = np.asarray(kmax)[:first]
    for p in range(first, P):
        rows = k_grown[p * page:min(N, (p + 1) * page)]
        new_min[p] = rows.min(axis=0)
        new_max[p] = rows.max(axis=0)
    return new_min, new_max
