"""Benchmark of cached block-diffusion attention (FlashBlock) on B200.

One step = one denoising step of one attention layer: the reuse gate, the
prefix (out-of-block) pass when the gate says recompute, the in-block pass and
the log-space merge -- the two C-ABI calls fb_prefix_attn(gate) and
fb_block_merge that make up fb_step.  Steps follow the seeded schedule of the
workload (16 steps per block for the dLM-like layer; step 0 of each block
recomputes), so the reported rate mixes recompute and reuse steps as the
method does.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Prints one JSON line (rank 0).  Under torchrun every rank runs its own replica
of the workload (weak scaling, no collective on the data path); the timed
region is bracketed by a barrier and a device synchronise and the slowest
rank's time is reported.
"""
from __future__ import annotations

import argparse
import hashlib
from typing import Optional
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from block_diffusion_attention_prefix_b200 import workloads as W  # noqa: E402

METRIC = "block-attention steps/sec and achieved HBM GB/s (% of B200 peak) vs context length"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0  # profiling recipe figures for this pool when no measurement exists
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


_READ_PEAK = {}


def read_peak_gbs(dev, gib: int = 4, reps: int = 5):
    """Read-only streaming bandwidth of this GPU, measured here: a sum over `gib` GiB
    of fp32 (torch's reduction kernel, 16-byte loads), best of `reps` with the events
    on the current stream.  A kernel that only reads (the prefix pass) can exceed the
    copy bandwidth of MEASURED_PEAKS.json, whose bytes are half writes; this figure
    is reported beside it, not instead of it."""
    key = str(dev)
    if key in _READ_PEAK:
        return _READ_PEAK[key]
    x = torch.ones((gib << 28,), device=dev, dtype=torch.float32)
    out = torch.empty((), device=dev, dtype=torch.float32)
    torch.sum(x, dim=0, out=out)
    best = 0.0
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch.sum(x, dim=0, out=out)
        e1.record()
        torch.cuda.synchronize()
        best = max(best, x.numel() * 4 / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    del x
    torch.cuda.empty_cache()
    _READ_PEAK[key] = best
    return best


def tensor_roofline(tflops: float) -> dict:
    """Tensor roofline of a step whose launch is timed alone (L2 flushed between
    steps): against the measured burst cuBLAS bf16 figure, with the sustained one
    (a seconds-long loop under the power cap) beside it."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        burst, sustained, kind = float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    else:
        burst, sustained, kind = FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"
    return dict(bound="tensor", achieved=tflops, peak=burst, unit="TFLOP/s", frac=tflops / burst,
                peak_source=f"{kind} burst cuBLAS bf16 (MEASURED_PEAKS.json bf16_tflops)",
                frac_of_sustained=tflops / sustained)


# Sources each profiled kernel is built from (its own translation unit and the headers
# it includes): a committed DRAM-traffic figure stays valid while these are unchanged.
KERNEL_SOURCES = {
    "pass_bf16_kernel": ["prefix_bf16.cu", "fb_device.cuh", "fb_ptx.cuh", "fb_internal.h"],
    "pass_tc_kernel": ["flash_tc.cu", "fb_device.cuh", "fb_ptx.cuh", "fb_internal.h"],
}


def kernel_source_hash(kernel: Optional[str] = None) -> str:
    """sha256 (16 hex) of one kernel's sources, or of every CUDA source when None."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_diffusion_attention_prefix_b200", "csrc")
    files = KERNEL_SOURCES[kernel] if kernel else sorted(f for f in os.listdir(csrc) if f.endswith((".cu", ".cuh", ".h")))
    for f in files:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per launch of the profiled kernel from the committed ncu summary,
    or None when the summary is absent or was taken on other sources of that kernel.
    A long-context length without its own summary takes the long_200k capture scaled
    by the algorithmic bytes of a recompute launch (the traffic is the prefix K/V
    read once, so it grows in proportion)."""
    own = os.path.join(ROOT, "profiles", f"prefix_pass_{workload}.md")
    ref = "long_200k" if workload.startswith("long_") else workload
    path = own if os.path.exists(own) else os.path.join(ROOT, "profiles", f"prefix_pass_{ref}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    kernel = vals.get("kernel")
    if kernel not in KERNEL_SOURCES or vals.get("kernel_source_sha") != kernel_source_hash(kernel):
        return None
    try:
        traffic = float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None
    if path != own:
        traffic *= step_bytes(W.get(workload))[0] / step_bytes(W.get(ref))[0]
    return traffic


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: record that no clocks were sampled
            self._nv = None
            self.error = str(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
                reasons = fn(self._h)
                self.samples.append((mhz, reasons))
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "nvml unavailable" if self._nv is None else "nvml"}
        mhz = [m for m, _ in self.samples]
        seen = set()
        for _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    seen.add(name)
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": sorted(seen),
                "samples": len(mhz), "source": "nvml"}


# ----------------------------------------------------------------------------- ranks


def replica_seed(seed: int, rank: int) -> int:
    """Each rank runs its own replica of the workload, drawn from its own seed."""
    return seed + rank


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's timed milliseconds (every rank gets it)."""
    if world <= 1:
        return ms
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, steps_per_rank: int, t_max_ms: float) -> float:
    """Whole-job steps/s: all ranks' steps over the slowest rank's time."""
    return world * steps_per_rank / (t_max_ms / 1e3)


# ----------------------------------------------------------------------------- device arm


class L2Flush:
    """Evicts the step's data from L2 between timed steps: writes a buffer larger
    than L2, then reads another one.  The read evicts the dirty lines of the write
    (their write-back happens here, outside the timed step), so the next step
    starts with an L2 full of clean, unrelated lines -- as after the other layers'
    attention in a model -- instead of paying ~126 MB of write-back itself."""

    def __init__(self, dev):
        self.w = torch.empty((L2_FLUSH_BYTES,), device=dev, dtype=torch.uint8)
        self.r = torch.ones((L2_FLUSH_BYTES // 4,), device=dev, dtype=torch.float32)
        self.sink = torch.empty((), device=dev, dtype=torch.float32)

    def __call__(self):
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.sink)


def step_bytes(w: W.Workload, batch: Optional[int] = None):
    """(recompute, reuse) algorithmic bytes of one dense step: what the fused step
    kernel must move for `batch` problems (default: the workload's batch).

    Recompute: prefix K and V, Q, the block's K and V, the cache rows written
    (A_out and L_out, fp32) and the output (A_full in the dtype, L_full fp32).
    Reuse: the same without the prefix K/V, with the cache read instead of written.
    """
    b = w.batch if batch is None else batch
    q = b * w.h_q * w.block * w.head_dim * w.elem_bytes
    kvb = 2 * b * w.h_kv * w.block * w.head_dim * w.elem_bytes
    cache = b * w.h_q * w.block * (w.head_dim + 1) * 4
    out = b * w.h_q * w.block * (w.head_dim * w.elem_bytes + 4)
    prefix = w.prefix_bytes() // w.batch * b
    return prefix + q + kvb + cache + out, q + kvb + cache + out


class DeviceWorkload:
    """The workload's inputs resident in HBM and the layer state, stepped through libfb."""

    def __init__(self, fb, w: W.Workload, seed: int, kv=None):
        self.fb, self.w = fb, w
        dev = torch.device("cuda")
        k, v = W.prefix_kv(w, seed) if kv is None else kv
        self.k, self.v = k.to(dev), v.to(dev)
        del k, v
        self.sched = []
        for s in W.block_schedule(w, seed):
            self.sched.append(dict(
                q=s.q.to(dev), k_blk=s.k_blk.to(dev), v_blk=s.v_blk.to(dev), mask=s.mask.to(dev),
                sim=None if s.sim is None else s.sim.to(dev), first=s.first,
                host=s))
        self.shape = fb.make_shape(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, w.n_prefix, w.dtype)
        f32 = dict(device=dev, dtype=torch.float32)
        self.a_out = torch.zeros((w.batch, w.h_q, w.block, w.head_dim), **f32)
        self.l_out = torch.full((w.batch, w.h_q, w.block), float("-inf"), **f32)
        self.a_full = torch.zeros((w.batch, w.h_q, w.block, w.head_dim), device=dev, dtype=w.torch_dtype)
        self.l_full = torch.zeros((w.batch, w.h_q, w.block), **f32)
        self.sparse_layer = None
        self.losa = w.losa_delta is not None
        if w.page_size:
            n_sel = sparse_n_select(w)
            if self.losa:
                self.sparse_layer = fb.LosaLayer(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, self.k, self.v,
                                                 n_sel, w.losa_delta, w.page_size)
            else:
                self.sparse_layer = fb.SparseResidualLayer(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, self.k,
                                                           self.v, n_sel, w.page_size)
            self.ws = self.sparse_layer.ws
        else:
            n = fb.fb_workspace_bytes(self.shape)
            self.ws = torch.zeros(((n + 15) // 16 * 16,), device=dev, dtype=torch.uint8)
        self.gates = [fb.make_gate(s["mask"], s["first"], w.tau, s["sim"], w.gamma or 0.0) for s in self.sched]

    def launches_per_step(self) -> int:
        # fb_step is one fused launch for blocks of up to 64 tokens; larger blocks
        # take the prefix pass, the gate record and the in-block pass.  The sparse
        # step is the page estimate, the top-k and the sparse pass.
        if self.sparse_layer is not None:
            return 3
        return 1 if self.w.block <= 64 else 3

    def entry(self, lib):
        if self.losa:  # the marshalled arguments start with the entry point of that step
            return lambda fn, *a: fn(*a)
        return lib.fb_sparse_step if self.sparse_layer is not None else lib.fb_step

    def step_args(self, i: int, dec_M, dec_reuse, tau_override=None):
        """Marshalled ctypes arguments of fb_step for schedule position i."""
        import ctypes
        fb, s = self.fb, self.sched[i % len(self.sched)]
        tau = self.w.tau if tau_override is None else tau_override
        g = fb.make_gate(s["mask"], s["first"], tau, s["sim"], self.w.gamma or 0.0)
        vp = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        if self.losa:
            lay, lib = self.sparse_layer, fb.load()
            pos = i % len(self.sched)
            if s["first"]:  # dense first step into the LoSA cache
                g = fb.make_gate(s["mask"], True, 1)
                args = (lib.fb_step, ctypes.byref(self.shape), vp(s["q"]), vp(self.k), vp(self.v), vp(s["k_blk"]),
                        vp(s["v_blk"]), ctypes.byref(g), vp(lay.a_res), vp(lay.l_res), vp(self.a_full),
                        vp(self.l_full), vp(dec_M), vp(dec_reuse), vp(lay.dense_ws), lay.dense_ws.numel(), stream)
                return args, g
            # tau_override=0 asks for the no-reuse reference: every token active (plain sparse attention)
            delta = float("-inf") if tau_override == 0 else self.w.losa_delta
            prev = self.sched[pos - 1]["q"]
            args = (lib.fb_losa_step, ctypes.byref(self.shape), vp(s["q"]), vp(prev), vp(self.k), vp(self.v),
                    vp(s["k_blk"]), vp(s["v_blk"]), ctypes.c_float(delta), ctypes.byref(lay.sparse),
                    vp(self.a_full), vp(self.l_full), vp(lay.mse), vp(lay.active), vp(self.ws), self.ws.numel(),
                    stream)
            return args, g
        if self.sparse_layer is not None:
            sl = self.sparse_layer
            args = (ctypes.byref(self.shape), vp(s["q"]), vp(self.k), vp(self.v), vp(s["k_blk"]), vp(s["v_blk"]),
                    ctypes.byref(g), ctypes.byref(sl.sparse), vp(self.a_full), vp(self.l_full), vp(dec_M),
                    vp(dec_reuse), vp(self.ws), self.ws.numel(), stream)
            return args, g
        args = (ctypes.byref(self.shape), vp(s["q"]), vp(self.k), vp(self.v), vp(s["k_blk"]), vp(s["v_blk"]),
                ctypes.byref(g), vp(self.a_out), vp(self.l_out), vp(self.a_full), vp(self.l_full), vp(dec_M),
                vp(dec_reuse), vp(self.ws), self.ws.numel(), stream)
        return args, g

    def union_density(self):
        """Fraction of prefix pages in the union of each KV group's selections (KV inflation)."""
        if self.sparse_layer is None:
            return None
        u = self.sparse_layer.union_bits.cpu().numpy().astype("uint32")
        ones = sum(bin(int(x)).count("1") for x in u.reshape(-1))
        return ones / (u.shape[0] * u.shape[1] * self.sparse_layer.n_pages)

    def algorithmic_bytes(self):
        if self.sparse_layer is not None:
            return self.sparse_algorithmic_bytes()
        return self.dense_algorithmic_bytes()

    def sparse_algorithmic_bytes(self):
        """(recompute, reuse) bytes of a sparse step: recompute reads all prefix K/V,
        the page bounds and Q and writes the residual and the output; reuse reads the
        union pages of each KV group (measured after the run) plus Q, the residual and
        the block, and writes the output."""
        w = self.w
        q = w.batch * w.h_q * w.block * w.head_dim * w.elem_bytes
        kvb = 2 * w.batch * w.h_kv * w.block * w.head_dim * w.elem_bytes
        res = w.batch * w.h_q * w.block * (w.head_dim + 1) * 4
        out = w.batch * w.h_q * w.block * (w.head_dim * w.elem_bytes + 4)
        bounds = 2 * w.batch * w.h_kv * w.head_dim * self.sparse_layer.n_pages * w.elem_bytes
        dens = self.union_density() or 1.0
        return (w.prefix_bytes() + bounds + q + kvb + res + out,
                int(w.prefix_bytes() * dens) + q + kvb + res + out)

    def dense_algorithmic_bytes(self):
        return step_bytes(self.w)


def batched_reuse(fb, w: W.Workload, flush, reps: int = 20, n_prefix: int = 64,
                  target_bytes: int = 192 << 20, max_problems: int = 4096):
    """Reuse steps of many independent problems in one fb_step launch (the batch
    dimension: layers x batch elements of the workload's shapes), so that the reuse
    path is seen streaming rather than launch-bound.  A reuse step reads no prefix
    K/V, so a short prefix (n_prefix tokens, allocated) stands in for it; the caches
    hold finite synthetic values and every step reuses (first_step = 0,
    tau = B + 1 > M).  Bytes per problem are the reuse step's algorithmic bytes (Q,
    the block's K/V, the cache read, A_full and L_full written)."""
    if w.block > 64 or w.page_size or w.losa_delta is not None:
        return None
    dev = torch.device("cuda")
    per = step_bytes(w, batch=1)[1]
    P = max(1, min(max_problems, -(-target_bytes // per)))
    g = torch.Generator(device=dev).manual_seed(1234)
    rnd = lambda *sh: torch.randn(sh, device=dev, generator=g).to(w.torch_dtype)  # noqa: E731
    q, kb, vb = rnd(P, w.h_q, w.block, w.head_dim), rnd(P, w.h_kv, w.block, w.head_dim), rnd(P, w.h_kv, w.block,
                                                                                            w.head_dim)
    k, v = rnd(P, w.h_kv, n_prefix, w.head_dim), rnd(P, w.h_kv, n_prefix, w.head_dim)
    mask = torch.ones((P, w.block), device=dev, dtype=torch.uint8)
    f32 = dict(device=dev, dtype=torch.float32)
    a_out = torch.randn((P, w.h_q, w.block, w.head_dim), device=dev, generator=g)
    l_out = torch.randn((P, w.h_q, w.block), device=dev, generator=g)
    a_full = torch.zeros((P, w.h_q, w.block, w.head_dim), device=dev, dtype=w.torch_dtype)
    l_full = torch.zeros((P, w.h_q, w.block), **f32)
    dM = torch.zeros((P,), device=dev, dtype=torch.int32)
    dR = torch.zeros((P, w.h_q), device=dev, dtype=torch.uint8)
    sh = fb.make_shape(P, w.h_q, w.h_kv, w.head_dim, w.block, n_prefix, w.dtype)
    n = fb.fb_workspace_bytes(sh)
    ws = torch.zeros(((n + 15) // 16 * 16,), device=dev, dtype=torch.uint8)
    fb.fb_workspace_init(ws)
    gate = fb.make_gate(mask, False, w.block + 1)
    for _ in range(3):
        fb.fb_step(sh, q, k, v, kb, vb, gate, a_out, l_out, a_full, l_full, dM, dR, ws)
    ev = []
    for _ in range(reps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fb.fb_step(sh, q, k, v, kb, vb, gate, a_out, l_out, a_full, l_full, dM, dR, ws)
        e1.record()
        ev.append((e0, e1))
    torch.cuda.synchronize()
    if not bool(dR.bool().all()):
        raise RuntimeError("batched reuse: a problem recomputed")
    us = statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3
    hbm, _ = peaks()
    gbs = P * per / (us * 1e-6) / 1e9
    out = dict(problems=P, n_prefix=n_prefix, bytes_per_launch=P * per, us=us, gbs=gbs, frac=gbs / hbm,
               note="reuse steps of P independent problems in one fb_step launch (median of "
                    f"{reps}, L2 flushed between); a reuse step reads no prefix K/V")
    del q, kb, vb, k, v, a_out, l_out, a_full, l_full, ws
    torch.cuda.empty_cache()
    return out


def device_arm(args, rank, world, w: Optional[W.Workload] = None, kv=None, extras: bool = True):
    """One workload through libfb on this rank's GPU.  `kv`: the prefix K/V already
    drawn on the host (else drawn here); `extras`: also measure the batched reuse
    view (independent of the prefix length)."""
    from block_diffusion_attention_prefix_b200 import fb
    fb.load()
    w = W.get(args.workload) if w is None else w
    dw = DeviceWorkload(fb, w, seed=replica_seed(args.seed, rank), kv=kv)
    K, Wm = args.steps, args.warmup
    dev = torch.device("cuda")
    flush = L2Flush(dev)
    dec_M = torch.zeros((K, w.batch), device=dev, dtype=torch.int32)
    dec_R = torch.zeros((K, w.batch, w.h_q), device=dev, dtype=torch.uint8)
    wdM = torch.zeros((w.batch,), device=dev, dtype=torch.int32)
    wdR = torch.zeros((w.batch, w.h_q), device=dev, dtype=torch.uint8)
    fb.fb_workspace_init(dw.ws)
    lib = fb.load()
    npos = len(dw.sched)
    # pre-marshalled fb_step arguments per schedule position (the timed steps write
    # their decisions to per-step rows of dec_M / dec_R)
    step_fn = dw.entry(lib)
    warm = [dw.step_args(i, wdM, wdR) for i in range(npos)]
    for i in range(Wm):
        flush()
        st = step_fn(*warm[i % npos][0])
        assert st == 0, fb.fb_status_string(st)
    torch.cuda.synchronize()
    start = Wm  # continue the schedule where warm-up stopped
    timed = [dw.step_args(start + i, dec_M[i], dec_R[i]) for i in range(K)]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    bad = 0
    with ClockSampler(torch.cuda.current_device()) as clocks:
        t0 = time.perf_counter()
        for i in range(K):
            flush()                      # L2 flush between timed steps (outside the events)
            evs[i][0].record()
            bad |= step_fn(*timed[i][0])
            evs[i][1].record()
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
    if bad:
        raise RuntimeError("fb_step failed inside the timed region")
    if world > 1:
        torch.distributed.barrier()
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    reuse = dec_R.cpu().numpy().astype(bool)            # [K, b, H_q]
    recompute_steps = [i for i in range(K) if not reuse[i].all()]
    reuse_steps = [i for i in range(K) if reuse[i].all()]
    total_ms = sum(step_ms)
    t_max = max_over_ranks(total_ms, world, dev)
    value = weak_scaling_value(world, K, t_max)
    hbm, peak_kind = peaks()
    alg, alg_reuse = dw.algorithmic_bytes()
    rec_ms = [step_ms[i] for i in recompute_steps]
    achieved = (alg * len(rec_ms)) / (sum(rec_ms) / 1e3) / 1e9 if rec_ms else None
    losa = None
    if dw.losa:
        # Dense first steps vs LoSA steps; the roofline is taken over the LoSA steps with
        # each schedule position's own bytes (its active rows' union pages), counted in an
        # untimed replay of the schedule (positions are deterministic).
        firsts = [dw.sched[(start + i) % npos]["first"] for i in range(K)]
        recompute_steps = [i for i in range(K) if firsts[i]]
        reuse_steps = [i for i in range(K) if not firsts[i]]
        lay = dw.sparse_layer
        q_b = w.batch * w.h_q * w.block * w.head_dim * w.elem_bytes
        kvb = 2 * w.batch * w.h_kv * w.block * w.head_dim * w.elem_bytes
        cache = w.batch * w.h_q * w.block * (w.head_dim + 1) * 4
        out = w.batch * w.h_q * w.block * (w.head_dim * w.elem_bytes + 4)
        page_kv = 2 * 16 * w.head_dim * w.elem_bytes
        pos_bytes, pos_union, pos_active = {}, {}, {}
        for pos in range(npos):
            st = step_fn(*warm[pos][0])
            assert st == 0, fb.fb_status_string(st)
            if not dw.sched[pos]["first"]:
                torch.cuda.synchronize()
                u = lay.union_bits.cpu().numpy().astype("uint32")
                pages = sum(bin(int(x)).count("1") for x in u.reshape(-1))
                pos_union[pos] = pages / (u.shape[0] * u.shape[1] * lay.n_pages)
                pos_active[pos] = float(lay.active.float().mean())
                pos_bytes[pos] = pages * page_kv + 2 * q_b + kvb + cache + out
        l_ms = [step_ms[i] for i in reuse_steps]
        l_bytes = [pos_bytes[(start + i) % npos] for i in reuse_steps]
        achieved = sum(l_bytes) / (sum(l_ms) / 1e3) / 1e9 if l_ms else None
        alg = int(sum(l_bytes) / len(l_bytes)) if l_bytes else 0
        rec_ms = l_ms
        losa = dict(delta=w.losa_delta, active_token_fraction=statistics.mean(pos_active.values()),
                    union_density_active_rows=statistics.mean(pos_union.values()),
                    losa_step_us=_mean_us(step_ms, reuse_steps), dense_first_step_us=_mean_us(step_ms,
                                                                                             recompute_steps))
    traffic = ncu_traffic(w.name)
    tensor = None
    if w.block > 64:
        # Large blocks (video): the passes are dense contractions.  FLOPs of a step =
        # 4 B D (N * heads that recompute + B * H_q)  (QK^T and PV, 2 flop per MAC).
        nrec = [int((~reuse[i]).sum()) for i in range(K)]
        flops = [4.0 * w.block * w.head_dim * (w.n_prefix * nrec[i] + w.block * w.h_q) * w.batch for i in range(K)]
        tflops = sum(flops) / (sum(step_ms) / 1e3) / 1e12
        tensor = tensor_roofline(tflops)
        tensor.update(flops_per_step_mean=sum(flops) / K, traffic=None,
                      kernel="pass_tc_kernel (tcgen05: prefix pass of recomputing heads + in-block pass)")

    # dense-recompute reference (standard block diffusion): gate forced to recompute
    dense_ms = []
    if args.dense_steps > 0:
        dense = [dw.step_args(i, wdM, wdR, tau_override=0) for i in range(args.dense_steps)]
        evd = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.dense_steps)]
        for i in range(args.dense_steps):
            flush()
            evd[i][0].record()
            step_fn(*dense[i][0])
            evd[i][1].record()
        torch.cuda.synchronize()
        dense_ms = [e[0].elapsed_time(e[1]) for e in evd]

    # Launch floor: the same event pair around libfb's smallest kernel (the gate
    # alone: one CTA per batch element) after the same L2 flush.
    floor = []
    for i in range(64):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fb.fb_gate_eval(dw.shape, dw.gates[i % npos], wdM, wdR)
        e1.record()
        floor.append((e0, e1))
    torch.cuda.synchronize()
    floor_us = statistics.median(a.elapsed_time(b) for a, b in floor) * 1e3

    # Block transition (once per block, after its last step): fb_append_block of one
    # block into a cache with room, with the page-bound refresh in sparse mode.
    n0, cap = 64, 64 + w.block
    kc = torch.zeros((w.batch, w.h_kv, cap, w.head_dim), device=dev, dtype=w.torch_dtype)
    vc = torch.zeros_like(kc)
    kb = torch.randn((w.batch, w.h_kv, w.block, w.head_dim), device=dev).to(w.torch_dtype)
    tsh = fb.make_shape(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, n0, w.dtype, kv_head_stride=cap * w.head_dim)
    kmn = kmx = None
    if dw.sparse_layer is not None:
        kmn = torch.zeros((w.batch, w.h_kv, w.head_dim, fb.fb_page_cap(tsh)), device=dev, dtype=w.torch_dtype)
        kmx = torch.zeros_like(kmn)
    trans = []
    for i in range(32):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fb.fb_append_block(tsh, kc, vc, kb, kb, 16, kmn, kmx)
        e1.record()
        trans.append((e0, e1))
    torch.cuda.synchronize()
    trans_us = statistics.median(a.elapsed_time(b) for a, b in trans) * 1e3

    # Per-head similarity estimate (gamma workloads): fb_head_similarity over the
    # block's queries and a reference block, as the estimated gate would run it.
    sim_us = sim_gbs = None
    if w.gamma is not None:
        qa = torch.randn((w.batch, w.h_q, w.block, w.head_dim), device=dev).to(w.torch_dtype)
        qb = torch.randn_like(qa)
        sim_out = torch.zeros((w.batch, w.h_q), device=dev)
        ssh = fb.make_shape(w.batch, w.h_q, w.h_kv, w.head_dim, w.block, w.n_prefix, w.dtype)
        nb = fb.fb_similarity_workspace_bytes(ssh)
        sws = torch.zeros(((nb + 15) // 16 * 16,), device=dev, dtype=torch.uint8)
        ev = []
        for i in range(20):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fb.fb_head_similarity(ssh, qa, qb, sim_out, sws)
            e1.record()
            ev.append((e0, e1))
        torch.cuda.synchronize()
        sim_us = statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3
        sim_gbs = 2 * qa.numel() * qa.element_size() / (sim_us * 1e-6) / 1e9

    reuse_batched = batched_reuse(fb, w, flush) if extras else None
    read_peak = read_peak_gbs(dev)
    reuse_ms = [step_ms[i] for i in reuse_steps]
    roofline_reuse = None
    if reuse_ms and not dw.losa:
        gbs = alg_reuse * len(reuse_ms) / (sum(reuse_ms) / 1e3) / 1e9
        roofline_reuse = dict(bound="launch", achieved=gbs, peak=hbm, unit="GB/s", frac=gbs / hbm,
                              alg_bytes_per_launch=alg_reuse, launches=len(reuse_ms),
                              avg_launch_us=sum(reuse_ms) / len(reuse_ms) * 1e3, launch_floor_us=floor_us,
                              note="a single reuse step reads no prefix K/V (Q, block K/V, cache, output only): "
                                   "launch bound; breakdown.reuse_batched is its HBM-bound view")
    e2e = e2e_arm(fb, dw, K, Wm) if (args.e2e and dw.sparse_layer is None) else None
    res = dict(
        metric=METRIC, value=value, unit="steps/s", n_gpus=world, steps=K, warmup=Wm,
        ms_per_step=t_max / K, higher_is_better=True, scaling="weak", vs_baseline=None,
        dtype=w.dtype, data="synthetic",
        config=dict(workload=w.name, description=w.description, batch=w.batch, h_q=w.h_q, h_kv=w.h_kv,
                    head_dim=w.head_dim, block=w.block, n_prefix=w.n_prefix, steps_per_block=w.steps,
                    tau=w.tau, gamma=w.gamma, seed=args.seed,
                    l2="flushed between timed steps, outside the step events: 256 MiB write then 256 MiB read "
                       "(the read evicts the write's dirty lines)",
                    parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
        roofline=dict(bound="hbm", kernel=("LoSA step (token score + page estimate + top-k + sparse_pass_kernel), "
                                           "LoSA steps" if dw.losa else
                                           "sparse step (page estimate + top-k + sparse_pass_kernel), recompute steps"
                                           if dw.sparse_layer is not None else
                                           (("pass_tc_kernel" if w.group * w.block > 16 and w.head_dim == 128
                                             else "pass_bf16_kernel") if w.dtype == "bf16" else "pass_f32_kernel")
                                           + (" (fused step: gate + prefix split-KV pass + in-block + merge), "
                                              "recompute launches" if w.block <= 64 else " (prefix split-KV pass)")),
                      achieved=achieved, peak=hbm, unit="GB/s",
                      frac=(achieved / hbm) if achieved else None,
                      peak_source=f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                      frac_of_8tbs=(achieved / 8000.0) if achieved else None,
                      read_peak=read_peak, frac_of_read_peak=(achieved / read_peak) if achieved else None,
                      alg_bytes_per_launch=alg, launches=len(rec_ms),
                      avg_launch_us=(sum(rec_ms) / len(rec_ms) * 1e3) if rec_ms else None,
                      traffic=traffic),
        breakdown=dict(recompute_steps=len(recompute_steps), reuse_steps=len(reuse_steps),
                       recompute_heads_per_step=float((~reuse).sum()) / K,
                       recompute_step_us=_mean_us(step_ms, recompute_steps),
                       reuse_step_us=_mean_us(step_ms, reuse_steps),
                       reuse_step_alg_bytes=alg_reuse,
                       roofline_reuse=roofline_reuse,
                       reuse_batched=reuse_batched,
                       launch_floor_us=floor_us,
                       block_transition_us=trans_us,
                       sim_estimator_us=sim_us, sim_estimator_gbs=sim_gbs,
                       dense_recompute_step_us=(statistics.mean(dense_ms) * 1e3) if dense_ms else None,
                       dense_steps_per_s=(1e3 / statistics.mean(dense_ms)) if dense_ms else None,
                       wall_s=wall),
        gpu_launches=(sum(1 if dw.sched[(start + i) % npos]["first"] else 4 for i in range(K)) if dw.losa
                      else dw.launches_per_step() * K),
        losa=losa,
        sparse=None if (dw.sparse_layer is None or dw.losa) else dict(
            n_select=dw.sparse_layer.sparse.n_select, pages=dw.sparse_layer.n_pages, union_density=dw.union_density(),
            reuse_step_gbs=(alg_reuse * len(reuse_steps)) / (sum(step_ms[i] for i in reuse_steps) / 1e3) / 1e9
            if reuse_steps else None),
        clocks=clocks.summary(),
        kernel_source_sha=kernel_source_hash(),
    )
    if tensor is not None:
        res["roofline_hbm"] = res["roofline"]
        res["roofline"] = tensor
    if e2e:
        res["e2e"] = e2e
    return res


def sparse_n_select(w: W.Workload) -> int:
    """k = ceil(density * pages), density read as the exact decimal it is written as."""
    from fractions import Fraction
    pages = (w.n_prefix + w.page_size - 1) // w.page_size
    return min(pages, max(1, math.ceil(Fraction(str(w.density)) * pages)))


def _mean_us(ms, idx):
    return statistics.mean(ms[i] for i in idx) * 1e3 if idx else None


def e2e_arm(fb, dw, K, Wm):
    """Same metric through fb_step with the step's inputs in pinned host memory.

    Every step copies its inputs host->device (one copy of a packed pinned buffer:
    q, the block's K and V, the mask, the similarity), runs fb_step (arguments
    marshalled once per schedule position) and copies A_full and the decisions back
    (one copy of a packed device buffer).  The host runs one step ahead: it waits for
    step i's result before reusing its host output buffer at step i + 2, and the
    timed region ends when every step's result is on the host."""
    import ctypes
    w = dw.w
    dev = torch.device("cuda")
    names = ("q", "k_blk", "v_blk", "mask", "sim")

    def seg(t):  # bytes of a segment, 16-byte aligned
        return (t.numel() * t.element_size() + 15) // 16 * 16

    s0 = dw.sched[0]["host"]
    proto = {"q": s0.q, "k_blk": s0.k_blk, "v_blk": s0.v_blk, "mask": s0.mask, "sim": s0.sim}
    offs, off = {}, 0
    for n in names:
        if proto[n] is not None:
            offs[n] = off
            off += seg(proto[n])
    in_bytes = off
    hosts = []
    for s in dw.sched:
        h = s["host"]
        buf = torch.zeros((in_bytes,), dtype=torch.uint8).pin_memory()
        for n in names:
            t = getattr(h, n)
            if t is not None:
                raw = t.contiguous().view(torch.uint8).reshape(-1)
                buf[offs[n]:offs[n] + raw.numel()].copy_(raw)
        hosts.append((buf, h.first))
    d_in = torch.empty((in_bytes,), dtype=torch.uint8, device=dev)

    def view(n):
        t = proto[n]
        nb = t.numel() * t.element_size()
        return d_in[offs[n]:offs[n] + nb].view(t.dtype).view(t.shape)
    dv = {n: (view(n) if n in offs else None) for n in names}
    # outputs packed: A_full (dtype) | dec_M int32 | dec_reuse uint8
    a_nb = dw.a_full.numel() * dw.a_full.element_size()
    m_off = (a_nb + 15) // 16 * 16
    r_off = m_off + (w.batch * 4 + 15) // 16 * 16
    out_bytes = r_off + (w.batch * w.h_q + 15) // 16 * 16
    d_out = torch.zeros((out_bytes,), dtype=torch.uint8, device=dev)
    a_full = d_out[:a_nb].view(dw.a_full.dtype).view(dw.a_full.shape)
    dM = d_out[m_off:m_off + w.batch * 4].view(torch.int32)
    dR = d_out[r_off:r_off + w.batch * w.h_q]
    ring = [torch.empty((out_bytes,), dtype=torch.uint8).pin_memory() for _ in range(2)]
    events = [None, None]
    lib = fb.load()
    vp = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stream = torch.cuda.current_stream()
    cs = ctypes.c_void_p(stream.cuda_stream)
    calls = []
    for (buf, first) in hosts:
        g = fb.make_gate(dv["mask"], first, w.tau, dv["sim"], w.gamma or 0.0)
        args = (ctypes.byref(dw.shape), vp(dv["q"]), vp(dw.k), vp(dw.v), vp(dv["k_blk"]), vp(dv["v_blk"]),
                ctypes.byref(g), vp(dw.a_out), vp(dw.l_out), vp(a_full), vp(dw.l_full), vp(dM), vp(dR),
                vp(dw.ws), dw.ws.numel(), cs)
        calls.append((buf, args, g))

    def one(i):
        buf, args, _ = calls[i % len(calls)]
        slot = i % 2
        if events[slot] is not None:
            events[slot].synchronize()  # step i - 2's result is on the host: its buffer is free
        d_in.copy_(buf, non_blocking=True)
        st = lib.fb_step(*args)
        if st != 0:
            raise RuntimeError(fb.fb_status_string(st))
        ring[slot].copy_(d_out, non_blocking=True)
        ev = torch.cuda.Event()
        ev.record(stream)
        events[slot] = ev

    for i in range(Wm):
        one(i)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(K):
        one(Wm + i)
    torch.cuda.synchronize()  # every step's result is on the host
    el = time.perf_counter() - t0
    kv_bytes = w.prefix_bytes()
    return dict(value=K / el, unit="steps/s", h2d_bytes_per_step=in_bytes, d2h_bytes_per_step=out_bytes,
                l2=f"not flushed between steps (wall clock of back-to-back steps); the prefix K/V hold "
                   f"{kv_bytes / 1e6:.0f} MB against a 126 MB L2" + (", so recompute steps stream them from HBM"
                                                                       if kv_bytes > 4 * (126 << 20) else
                                                                       ", so part of them can stay resident"),
                note="wall clock per step incl. one pinned H2D copy of the step's packed inputs, fb_step, one "
                     "D2H copy of A_full + decisions; the host runs one step ahead (waits for step i's result "
                     "before reusing its output buffer at step i+2); prefix KV cache resident in HBM")


# ----------------------------------------------------------------------------- oracle arm


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_steps(w: W.Workload, seed: int, budget_s: float, max_steps: int, kv_groups: int, kv=None):
    """Time the CPU oracle's cached step on the workload, restricted to the first
    `kv_groups` KV-head groups (a bounded sample).  Returns (steps, seconds,
    scale) where scale converts the sample's time to a whole-layer step.  `kv`:
    the prefix K/V already drawn (else drawn here)."""
    from oracle import flashblock as OF
    from oracle import sparse as OS
    k, v = W.prefix_kv(w, seed) if kv is None else kv
    hk = min(kv_groups, w.h_kv)
    hq = hk * w.group
    kk = k[:, :hk].double().numpy()
    vv = v[:, :hk].double().numpy()
    del k, v
    if w.losa_delta is not None:
        from oracle import losa as OL
        lo = OL.LosaAttention(kk, vv, hq, 1 / math.sqrt(w.head_dim), w.page_size, w.density)
        prev = {}

        def losa_step(q, kb, vb, mask, first, tau, sim, gamma):
            r = lo.step(q, prev.get("q"), kb, vb, first, w.losa_delta)
            prev["q"] = q
            return r
        st = type("LosaStep", (), {"step": staticmethod(losa_step)})()
    elif w.page_size:
        sp = OS.SparseResidualAttention(kk, vv, hq, 1 / math.sqrt(w.head_dim), w.page_size, w.density)
        st = type("SparseStep", (), {"step": staticmethod(
            lambda q, kb, vb, mask, first, tau, sim, gamma: sp.step(q, kb, vb, mask, first, tau))})()
    else:
        st = OF.CachedBlockAttention(kk, vv, hq, 1 / math.sqrt(w.head_dim))
    sched = list(W.block_schedule(w, seed))
    conv = [(s.q[:, :hq].double().numpy(), s.k_blk[:, :hk].double().numpy(), s.v_blk[:, :hk].double().numpy(),
             s.mask.numpy(), s.first, None if s.sim is None else s.sim[:, :hq].numpy()) for s in sched]
    n, el = 0, 0.0
    while n < max_steps and (el < budget_s or n < 1):
        q, kb, vb, mask, first, sim = conv[n % len(conv)]
        t0 = time.perf_counter()
        st.step(q, kb, vb, mask, first, w.tau, sim, w.gamma or 0.0)
        el += time.perf_counter() - t0
        n += 1
    return n, el, w.h_kv / hk


def cpu_baseline(w, seed, budget_s=12.0, one_thread_budget_s=4.0, kv=None):
    """The float64 oracle on the host cores (all BLAS threads), plus the same sample
    with the BLAS pools held to one thread (`one_thread`)."""
    n, el, scale = oracle_steps(w, seed, budget_s, 10 ** 6, kv_groups=1, kv=kv)
    out = dict(value=n / (el * scale), unit="steps/s", cores=blas_threads(), kind="oracle",
               sample=f"{n} steps of the seeded schedule through the float64 oracle, 1 of {w.h_kv} KV-head "
                      f"groups ({w.group} query heads) at full prefix length; time x{scale:g} = whole layer")
    one = None
    if one_thread_budget_s > 0:
        try:
            from threadpoolctl import threadpool_limits
        except ImportError:
            threadpool_limits = None
        if threadpool_limits is not None:
            with threadpool_limits(limits=1):
                n1, el1, scale1 = oracle_steps(w, seed, one_thread_budget_s, 10 ** 6, kv_groups=1, kv=kv)
            one = dict(value=n1 / (el1 * scale1), unit="steps/s", cores=1, sample=f"{n1} steps, same sample")
    out["one_thread"] = one
    return out


def reference_arm(args):
    w = W.get(SWEEP[-1] if args.workload == "long_sweep" else args.workload)
    kv = W.prefix_kv(w, args.seed)
    _, _, _ = oracle_steps(w, args.seed, 0.0, max(1, min(args.warmup, 16)), kv_groups=1, kv=kv)
    n, el, scale = oracle_steps(w, args.seed, 1e9, args.steps, kv_groups=1, kv=kv)
    value = n / (el * scale)
    return dict(metric=METRIC, value=value, unit="steps/s", n_gpus=args.gpus, steps=n, warmup=args.warmup,
                ms_per_step=el * scale / n * 1e3, higher_is_better=True, scaling="weak", vs_baseline=None,
                dtype="f64", data="synthetic", impl="reference",
                config=dict(workload=w.name, description=w.description, batch=w.batch, h_q=w.h_q, h_kv=w.h_kv,
                            head_dim=w.head_dim, block=w.block, n_prefix=w.n_prefix, tau=w.tau,
                            l2="n/a (host)", parallelism="host cores"),
                cpu_baseline=dict(value=value, unit="steps/s", cores=blas_threads(), kind="oracle",
                                  sample=f"each step: the float64 oracle on 1 of {w.h_kv} KV-head groups at full "
                                         f"prefix length, time x{scale:g} = whole layer"),
                e2e=dict(value=value, unit="steps/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))


# ----------------------------------------------------------------------------- context-length sweep

# The metric is taken against context length: the long-context workloads at 100k,
# 200k, 400k and 800k prefix tokens, the top-level figures at the largest; the
# dLM-8B-like 32k layer rides along as a secondary record.
SWEEP = ("long_100k", "long_200k", "long_400k", "long_800k")
SWEEP_SECONDARY = ("dlm8b_b4",)


def sweep_entry(r: dict) -> dict:
    """The per-length summary of one workload's record."""
    bd, rf = r["breakdown"], r["roofline"]
    cb = r.get("cpu_baseline")
    return dict(
        workload=r["config"]["workload"], n_prefix=r["config"]["n_prefix"], steps_per_s=r["value"],
        ms_per_step=r["ms_per_step"], steps=r["steps"],
        roofline=dict(achieved=rf["achieved"], peak=rf["peak"], unit=rf["unit"], frac=rf["frac"],
                      frac_of_8tbs=rf.get("frac_of_8tbs"), frac_of_read_peak=rf.get("frac_of_read_peak"),
                      alg_bytes_per_launch=rf["alg_bytes_per_launch"],
                      launches=rf["launches"], avg_launch_us=rf["avg_launch_us"], traffic=rf.get("traffic")),
        roofline_reuse=bd.get("roofline_reuse"),
        recompute_steps=bd["recompute_steps"], reuse_steps=bd["reuse_steps"],
        recompute_step_us=bd["recompute_step_us"], reuse_step_us=bd["reuse_step_us"],
        dense_recompute_step_us=bd["dense_recompute_step_us"], dense_steps_per_s=bd["dense_steps_per_s"],
        e2e_steps_per_s=(r.get("e2e") or {}).get("value"),
        cpu_baseline=None if cb is None else dict(value=cb["value"], unit=cb["unit"], cores=cb["cores"],
                                                  sample=cb["sample"]),
        clocks=r.get("clocks"))


def sweep_arm(args, rank, world):
    """Every sweep length (and the secondary workloads) through device_arm; the
    top-level record is the largest length's, with one summary per length."""
    recs = {}
    for name in SWEEP + SWEEP_SECONDARY:
        w = W.get(name)
        kv = W.prefix_kv(w, replica_seed(args.seed, rank))
        r = device_arm(args, rank, world, w=w, kv=kv, extras=(name == SWEEP[-1]))
        if rank == 0 and world == 1 and args.cpu_baseline:
            r["cpu_baseline"] = cpu_baseline(w, args.seed, budget_s=5.0, one_thread_budget_s=2.0, kv=kv)
        del kv
        torch.cuda.empty_cache()
        recs[name] = r
    res = recs[SWEEP[-1]]
    res["config"]["sweep"] = list(SWEEP)
    res["sweep"] = [sweep_entry(recs[n]) for n in SWEEP]
    res["secondary"] = {n: sweep_entry(recs[n]) for n in SWEEP_SECONDARY}
    return res


# ----------------------------------------------------------------------------- context-parallel arm


def context_arm(args, rank, world):
    """--split context: the workload's prefix cut into `world` key ranges, one per
    rank (block_diffusion_attention_prefix_b200.context_parallel): every step each
    rank computes its range's partial, one all-gather exchanges the partials, and
    every rank merges them and finishes the step.  The whole job is one layer, so
    this is strong scaling: value = steps of the layer per second, timed as the
    slowest rank's summed step events."""
    from block_diffusion_attention_prefix_b200 import fb
    from block_diffusion_attention_prefix_b200.context_parallel import ContextParallelLayer, shard_range
    fb.load()
    w = W.get(SWEEP[-1] if args.workload == "long_sweep" else args.workload)
    if w.block > 64 or w.page_size or w.losa_delta is not None:
        raise SystemExit(f"--split context takes the dense small-block workloads, not {w.name}")
    dev = torch.device("cuda")
    n0, n1 = shard_range(w.n_prefix, world, rank)
    # this rank's range of the prefix, drawn on the device (seeded per rank); the
    # block's inputs are the same on every rank
    g = torch.Generator(device=dev).manual_seed(args.seed * 1_000_003 + rank)
    c = (0.5 * (0.5 + 1.5 * torch.rand(w.h_kv, generator=g, device=dev))).view(1, w.h_kv, 1, 1)
    shape = (w.batch, w.h_kv, n1 - n0, w.head_dim)
    k = (torch.randn(shape, generator=g, device=dev) * c).to(w.torch_dtype)
    v = (torch.randn(shape, generator=g, device=dev) * c).to(w.torch_dtype)
    sched = [dict(q=s.q.to(dev), k_blk=s.k_blk.to(dev), v_blk=s.v_blk.to(dev), mask=s.mask.to(dev), first=s.first)
             for s in W.block_schedule(w, args.seed)]
    layer = ContextParallelLayer(fb, w.batch, w.h_q, w.h_kv, w.head_dim, w.block, w.n_prefix, k, v, rank, world)
    flush = L2Flush(dev)
    K, Wm, npos = args.steps, args.warmup, len(sched)

    def one(i):
        s = sched[i % npos]
        layer.step(s["q"], s["k_blk"], s["v_blk"], s["mask"], s["first"], w.tau)

    for i in range(Wm):
        flush()
        one(i)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    reuse = []
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        for i in range(K):
            flush()
            evs[i][0].record()
            one(Wm + i)
            evs[i][1].record()
            reuse.append(layer.dec_reuse.clone())
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    t_max = max_over_ranks(sum(step_ms), world, dev)
    rec = [i for i in range(K) if not bool(reuse[i].bool().all())]
    re_ = [i for i in range(K) if bool(reuse[i].bool().all())]
    hbm, peak_kind = peaks()
    shard_bytes = 2 * w.batch * w.h_kv * (n1 - n0) * w.head_dim * w.elem_bytes
    rec_us = _mean_us(step_ms, rec)
    achieved = shard_bytes / (rec_us * 1e-6) / 1e9 if rec_us else None
    exch = world * layer.flat * 4
    return dict(
        metric=METRIC, value=K / (t_max / 1e3), unit="steps/s", n_gpus=world, steps=K, warmup=Wm,
        ms_per_step=t_max / K, higher_is_better=True, scaling="strong", vs_baseline=None, dtype=w.dtype,
        data="synthetic",
        config=dict(workload=w.name, description=w.description, batch=w.batch, h_q=w.h_q, h_kv=w.h_kv,
                    head_dim=w.head_dim, block=w.block, n_prefix=w.n_prefix, tau=w.tau, seed=args.seed,
                    l2="flushed between timed steps, outside the step events",
                    parallelism=f"context x{world} (prefix key ranges of {n1 - n0} tokens on rank {rank})"),
        roofline=dict(bound="hbm", kernel="rank's recompute step: prefix pass over its key range + all-gather of "
                                          "the partials + merge + in-block", achieved=achieved, peak=hbm, unit="GB/s",
                      frac=achieved / hbm if achieved else None, peak_source=f"{peak_kind} copy bandwidth",
                      alg_bytes_per_launch=shard_bytes, traffic=None),
        breakdown=dict(recompute_steps=len(rec), reuse_steps=len(re_), recompute_step_us=rec_us,
                       reuse_step_us=_mean_us(step_ms, re_), exchange_bytes_per_step=exch,
                       note="every step runs the all-gather (the gate is evaluated on the device)"),
        gpu_launches=3 * K, clocks=clocks.summary(), kernel_source_sha=kernel_source_hash())


# ----------------------------------------------------------------------------- main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps per workload (default 200 for the long-context workloads, else 2000)")
    ap.add_argument("--warmup", type=int, default=32)
    ap.add_argument("--workload", default="long_sweep", choices=["long_sweep"] + sorted(W.WORKLOADS),
                    help="long_sweep (default): the context-length sweep 100k/200k/400k/800k, top-level "
                         "figures at 800k, dlm8b_b4 as a secondary record")
    ap.add_argument("--impl", default="fb", choices=["fb", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--dense-steps", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--split", default="replicas", choices=["replicas", "context"],
                    help="replicas (default): one replica of the workload per rank (weak scaling); context: the "
                         "prefix split over the ranks by key range (strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.steps is None:
        args.steps = 200 if args.workload == "long_sweep" or args.workload.startswith("long_") else 2000

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args)), flush=True)
        return

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    if args.split == "context":
        res = context_arm(args, rank, world)
    elif args.workload == "long_sweep":
        res = sweep_arm(args, rank, world)
    else:
        res = device_arm(args, rank, world)
        if rank == 0 and world == 1 and args.cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(W.get(args.workload), args.seed)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
