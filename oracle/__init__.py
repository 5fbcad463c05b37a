"""CPU oracle for cached block-diffusion attention (FlashBlock).

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, float64 restatement of
what the pages define.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it.  The product path
(``block_diffusion_attention_prefix_b200`` and ``libfb.so``) never imports,
links or calls anything here, and nothing here imports the product path: the
two share only the seeded input generators in
``block_diffusion_attention_prefix_b200.workloads``.

Sources (web pages; cited by title and section):
* "Technical summary: FlashBlock" (gist.science, paper 2602.05305; Italian,
  Korean and German versions agree), sections "1. Problem definition",
  "2. Methodology: FlashBlock / Core mechanism" (the split into J_in and J_out,
  the cached (A_out, L_out = log Z_out) and the log-space merge equation) and
  "Adaptive reuse strategies" (tau threshold, per-head gamma, sparse residual).
* "LoSA: Locality Aware Sparse Attention for Block-Wise Diffusion Language
  Models" (gist.science, paper 2604.12056), "1. The problem: KV inflation" and
  "2. Methodology" (first step of a block is dense; QUEST as the page selector).

Modules:
* :mod:`oracle.attention`  -- softmax attention over a key set as (A, L), and the merge.
* :mod:`oracle.flashblock` -- the tau / gamma gates and the stateful cached step.
* :mod:`oracle.sparse`     -- page bounds, top-k page selection and the residual split.
* :mod:`oracle.transition` -- the block transition: a finished block joins the prefix.
* :mod:`oracle.similarity` -- the per-head similarity estimate behind the gamma gate.
* :mod:`oracle.losa`       -- LoSA-style per-token reuse: active tokens sparse, stable tokens cached.

Pins: every function here is pinned by ``tests/test_oracle_*.py`` against
library routines (torch float64 SDPA, logsumexp, full sorts), closed forms and
hand-derived fixtures in ``tests/golden/``.  Model-level quality and tokens/s
figures from the pages are "parity unpinned" (they need trained weights).
"""
