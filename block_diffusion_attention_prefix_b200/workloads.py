"""Seeded synthetic workloads for cached block-diffusion attention.

This module only draws random inputs.  It holds none of the attention, merge
or gating arithmetic: the GPU path (through the C-ABI) and the CPU oracle both
consume the exact tensors produced here, so that parity compares the two
implementations on identical bytes.

Shapes follow the FlashBlock technical summary (gist.science paper 2602.05305,
"1. Problem definition" and "2. Methodology / Core mechanism"): a block of B
query tokens per step, a prefix KV cache of N tokens that the block attends to
(J_out) and the block's own B keys (J_in).  The pages give no input laws; the
recipes below are this library's readings:

* Q ~ N(0, 1).  Prefix and in-block K/V ~ N(0, 1) * 0.5 * c_g with a per-KV-head
  scale c_g ~ U(0.5, 2) (dLM, long-context, video and sparse workloads); the
  tiny fp32 workload uses plain N(0, 1).
* Step 0 of a block marks every token as updated (the block is new).  Later
  steps mark a random subset: either M ~ U{0..B} tokens at random positions
  (tiny fp32) or each token independently with p = 0.25, so that M ~ Bin(B, .25)
  (dLM-like).  Updated tokens get fresh q (all query heads) and fresh k/v (all
  KV heads); the others keep theirs bit for bit.
* Video: every block token is resampled every step, and a per-head cross-step
  similarity is drawn U(0.8, 1.0) per step.

Tensors are torch CPU tensors in the library's layouts:
Q [b, H_q, B, D], prefix K/V [b, H_kv, N, D], in-block K/V [b, H_kv, B, D],
mask uint8 [b, B], sim float32 [b, H_q].
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterator, Optional

import torch

__all__ = ["Workload", "WORKLOADS", "prefix_kv", "block_schedule", "Step", "get"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str                 # "f32" or "bf16"
    batch: int
    h_q: int
    h_kv: int
    head_dim: int
    block: int                 # B, queries per step
    n_prefix: int              # N, prefix tokens (J_out)
    steps: int                 # denoising steps per block
    tau: int                   # reuse iff M < tau (after step 0)
    gamma: Optional[float]     # per-head gate (video); None = no per-head gate
    mask_law: str              # "uniform_count" | "binomial" | "all"
    kv_head_scale: bool        # per-KV-head scale c_g ~ U(0.5, 2), times 0.5
    page_size: int = 0         # sparse workloads only
    density: float = 0.0       # sparse workloads only
    losa_delta: Optional[float] = None  # LoSA workloads: activity threshold on the locality score
    description: str = ""

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def prefix_bytes(self) -> int:
        """Bytes of prefix K and V for the whole batch."""
        return 2 * self.batch * self.h_kv * self.n_prefix * self.head_dim * self.elem_bytes


def _dlm(name, n, block, steps, **kw):
    return Workload(name=name, dtype="bf16", batch=1, h_q=32, h_kv=8, head_dim=128,
                    block=block, n_prefix=n, steps=steps, tau=block // 2, gamma=None,
                    mask_law="binomial", kv_head_scale=True, **kw)


WORKLOADS = {
    "tiny_f32": Workload(
        name="tiny_f32", dtype="f32", batch=1, h_q=2, h_kv=1, head_dim=64, block=4,
        n_prefix=1024, steps=8, tau=2, gamma=None, mask_law="uniform_count",
        kv_head_scale=False,
        description="tiny fp32: b=1, 2 q heads / 1 kv head, D=64, N=1024, B=4, 8 steps, tau=2"),
    "dlm8b_b4": _dlm("dlm8b_b4", 32768, 4, 16,
                     description="dLM-8B-like bf16 layer: b=1, H_q=32, H_kv=8, D=128, N=32768, "
                                 "B=4, 16 steps, M~Bin(4,.25), tau=2"),
    "dlm8b_b16": _dlm("dlm8b_b16", 32768, 16, 16,
                      description="dLM-8B-like bf16 layer: b=1, H_q=32, H_kv=8, D=128, N=32768, "
                                  "B=16, 16 steps, M~Bin(16,.25), tau=8"),
    "long_100k": _dlm("long_100k", 100_000, 4, 8, description="long context bf16, N=100000, B=4, 8 steps"),
    "long_200k": _dlm("long_200k", 200_000, 4, 8, description="long context bf16, N=200000, B=4, 8 steps"),
    "long_400k": _dlm("long_400k", 400_000, 4, 8, description="long context bf16, N=400000, B=4, 8 steps"),
    "long_800k": _dlm("long_800k", 800_000, 4, 8, description="long context bf16, N=800000, B=4, 8 steps"),
    "video": Workload(
        name="video", dtype="bf16", batch=1, h_q=12, h_kv=12, head_dim=128, block=3 * 1560,
        n_prefix=20 * 1560, steps=4, tau=3 * 1560 + 1, gamma=0.95, mask_law="all",
        kv_head_scale=True,
        description="video-diffusion-like bf16: b=1, 12 heads MHA, D=128, prefix 20x1560, "
                    "block 3x1560, 4 steps, sim~U(.8,1), gamma=0.95"),
    "sparse64k": _dlm("sparse64k", 65536, 4, 16, page_size=16, density=0.2,
                      description="sparse+residual bf16: dLM-8B-like shapes, N=65536, 16-token pages, "
                                  "density 0.2, B=4, 16 steps, tau=2"),
    "losa64k": _dlm("losa64k", 65536, 4, 16, page_size=16, density=0.2, losa_delta=0.01,
                    description="LoSA-style bf16: sparse64k shapes; after a dense first step, tokens whose "
                                "queries moved (score > 0.01) get sparse attention over their top 20% pages, "
                                "stable tokens reuse; union over active tokens only"),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def _gen(seed: int, stream: int) -> torch.Generator:
    # independent streams for prefix, per-step inputs and gate draws
    return torch.Generator().manual_seed((seed * 1_000_003 + stream * 7919) % (2**63 - 1))


def _kv_head_scale(w: Workload, seed: int) -> torch.Tensor:
    if not w.kv_head_scale:
        return torch.ones(w.h_kv)
    g = _gen(seed, 1)
    return 0.5 * (0.5 + 1.5 * torch.rand(w.h_kv, generator=g))


def prefix_kv(w: Workload, seed: int, n_prefix: Optional[int] = None):
    """Prefix K and V caches [b, H_kv, N, D] in the workload dtype."""
    n = w.n_prefix if n_prefix is None else n_prefix
    c = _kv_head_scale(w, seed).view(1, w.h_kv, 1, 1)
    g = _gen(seed, 2)
    shape = (w.batch, w.h_kv, n, w.head_dim)
    k = torch.randn(shape, generator=g).mul_(c).to(w.torch_dtype)
    v = torch.randn(shape, generator=g).mul_(c).to(w.torch_dtype)
    return k, v


@dataclasses.dataclass
class Step:
    index: int
    first: bool
    q: torch.Tensor        # [b, H_q, B, D]
    k_blk: torch.Tensor    # [b, H_kv, B, D]
    v_blk: torch.Tensor    # [b, H_kv, B, D]
    mask: torch.Tensor     # uint8 [b, B]; 1 = token updated at this step
    sim: Optional[torch.Tensor]  # float32 [b, H_q] or None


def block_schedule(w: Workload, seed: int, steps: Optional[int] = None) -> Iterator[Step]:
    """The seeded denoising-step schedule of one block (inputs only, no results)."""
    steps = w.steps if steps is None else steps
    g = _gen(seed, 3)
    c = _kv_head_scale(w, seed).view(1, w.h_kv, 1, 1)
    b, hq, hk, B, D = w.batch, w.h_q, w.h_kv, w.block, w.head_dim
    q = torch.randn((b, hq, B, D), generator=g).to(w.torch_dtype)
    kb = torch.randn((b, hk, B, D), generator=g).mul_(c).to(w.torch_dtype)
    vb = torch.randn((b, hk, B, D), generator=g).mul_(c).to(w.torch_dtype)
    for s in range(steps):
        if s == 0 or w.mask_law == "all":
            mask = torch.ones((b, B), dtype=torch.uint8)
        elif w.mask_law == "binomial":
            mask = (torch.rand((b, B), generator=g) < 0.25).to(torch.uint8)
        elif w.mask_law == "uniform_count":
            mask = torch.zeros((b, B), dtype=torch.uint8)
            for bi in range(b):
                m = int(torch.randint(0, B + 1, (1,), generator=g))
                pos = torch.randperm(B, generator=g)[:m]
                mask[bi, pos] = 1
        else:
            raise ValueError(w.mask_law)
        if s > 0:
            upd = mask.bool()
            if bool(upd.any()):
                nq = torch.randn((b, hq, B, D), generator=g).to(w.torch_dtype)
                nk = torch.randn((b, hk, B, D), generator=g).mul_(c).to(w.torch_dtype)
                nv = torch.randn((b, hk, B, D), generator=g).mul_(c).to(w.torch_dtype)
                sel_q = upd.view(b, 1, B, 1).expand_as(q)
                sel_k = upd.view(b, 1, B, 1).expand_as(kb)
                q = torch.where(sel_q, nq, q)
                kb = torch.where(sel_k, nk, kb)
                vb = torch.where(sel_k, nv, vb)
        sim = None
        if w.gamma is not None:
            sim = (0.8 + 0.2 * torch.rand((b, hq), generator=g)).to(torch.float32)
        yield Step(index=s, first=(s == 0), q=q.clone(), k_blk=kb.clone(), v_blk=vb.clone(),
                   mask=mask, sim=sim)


def generation_schedule(w: Workload, seed: int, blocks: int, steps: Optional[int] = None):
    """Several consecutive blocks (inputs only): a list per block of its denoising
    steps.  Block t draws from seed + 7919 * t; the block's keys and values as of its
    last step are what joins the prefix when the block is finished."""
    return [list(block_schedule(w, seed + 7919 * t, steps)) for t in range(blocks)]


def default_scale(head_dim: int) -> float:
    """Softmax temperature used when the caller passes 0: 1/sqrt(D)."""
    return 1.0 / math.sqrt(head_dim)
