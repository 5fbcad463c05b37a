"""ctypes binding of libfb.so (include/fb.h), argument marshalling only.

Every function here has the name of the C entry point it calls and forwards
torch tensors as raw device pointers plus the current torch CUDA stream.  All
computation happens in libfb's CUDA kernels; there is no fallback: if the
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "FBError", "Shape", "Gate", "load", "lib_path", "make_shape", "make_gate", "FB_F32", "FB_BF16",
    "fb_version", "fb_status_string", "fb_device_error", "fb_workspace_bytes", "fb_workspace_init",
    "fb_gate_eval", "fb_prefix_attn", "fb_prefix_attn_noalloc", "fb_block_attn", "fb_merge", "fb_merge_partials", "fb_exp2_fma",
    "fb_block_merge", "fb_step",
    "fb_page_minmax", "fb_append_block", "fb_similarity_workspace_bytes", "fb_head_similarity",
    "fb_refresh_reference", "fb_losa_step", "LosaLayer", "fb_sparse_workspace_bytes", "fb_sparse_select", "fb_sparse_step", "Sparse",
    "SparseResidualLayer", "CachedAttentionLayer", "EXPORTED",
]

FB_F32 = 0
FB_BF16 = 1

_HERE = os.path.dirname(os.path.abspath(__file__))


def lib_path() -> str:
    return os.environ.get("FB_LIBRARY", os.path.join(_HERE, "libfb.so"))


class FBError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: status {status} ({msg})")
        self.status = status


class Shape(ctypes.Structure):
    """struct fb_shape."""
    _fields_ = [("batch", ctypes.c_int32), ("h_q", ctypes.c_int32), ("h_kv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("n_prefix", ctypes.c_int64), ("kv_row_stride", ctypes.c_int64),
                ("kv_head_stride", ctypes.c_int64), ("scale", ctypes.c_float)]


class Gate(ctypes.Structure):
    """struct fb_gate (device pointers to the mask and optional head similarity)."""
    _fields_ = [("updated_mask", ctypes.c_void_p), ("head_sim", ctypes.c_void_p),
                ("first_step", ctypes.c_int32), ("tau", ctypes.c_int32), ("gamma", ctypes.c_float)]


class Sparse(ctypes.Structure):
    """struct fb_sparse (device pointers to the page bounds and the sparse state)."""
    _fields_ = [("page_size", ctypes.c_int32), ("n_select", ctypes.c_int32), ("kmin", ctypes.c_void_p),
                ("kmax", ctypes.c_void_p), ("sel_idx", ctypes.c_void_p), ("sel_bits", ctypes.c_void_p),
                ("union_bits", ctypes.c_void_p), ("a_res", ctypes.c_void_p), ("l_res", ctypes.c_void_p),
                ("a_sel", ctypes.c_void_p), ("l_sel", ctypes.c_void_p)]


_vp = ctypes.c_void_p
_sz = ctypes.c_size_t
_i = ctypes.c_int
_PS = ctypes.POINTER(Shape)
_PG = ctypes.POINTER(Gate)
_PSP = ctypes.POINTER(Sparse)

# name -> (restype, argtypes); the set of exported C-ABI symbols.
EXPORTED = {
    "fb_version": (_i, []),
    "fb_status_string": (ctypes.c_char_p, [_i]),
    "fb_device_error": (_i, [ctypes.POINTER(ctypes.c_int32)]),
    "fb_workspace_bytes": (_sz, [_PS]),
    "fb_workspace_init": (_i, [_vp, _sz, _vp]),
    "fb_gate_eval": (_i, [_PS, _PG, _vp, _vp, _vp]),
    "fb_prefix_attn": (_i, [_PS, _vp, _vp, _vp, _PG, _vp, _vp, _vp, _sz, _vp]),
    "fb_block_attn": (_i, [_PS, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "fb_merge": (_i, [_PS, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fb_block_merge": (_i, [_PS, _vp, _vp, _vp, _PG, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "fb_step": (_i, [_PS, _vp, _vp, _vp, _vp, _vp, _PG, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "fb_prefix_attn_noalloc": (_i, [_PS, _vp, _vp, _vp, _PG, _vp, _vp, _vp]),
    "fb_merge_partials": (_i, [_PS, _vp, ctypes.c_int64, _vp, ctypes.c_int64, _i, _PG, _vp, _vp, _vp]),
    "fb_exp2_fma": (_i, [_vp, _vp, ctypes.c_int64, _vp]),
    "fb_page_cap": (_i, [_PS, _i]),
    "fb_page_minmax": (_i, [_PS, _vp, _i, _vp, _vp, _vp]),
    "fb_append_block": (_i, [_PS, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp]),
    "fb_similarity_workspace_bytes": (_sz, [_PS]),
    "fb_head_similarity": (_i, [_PS, _vp, _vp, _vp, _vp, _sz, _vp]),
    "fb_refresh_reference": (_i, [_PS, _vp, _vp, _vp, _vp]),
    "fb_losa_step": (_i, [_PS, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _PSP, _vp, _vp, _vp, _vp, _vp, _sz,
                          _vp]),
    "fb_sparse_workspace_bytes": (_sz, [_PS, _i]),
    "fb_sparse_select": (_i, [_PS, _vp, _PG, _PSP, _vp, _sz, _vp]),
    "fb_sparse_step": (_i, [_PS, _vp, _vp, _vp, _vp, _vp, _PG, _PSP, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
}

_lib: Optional[ctypes.CDLL] = None


def load() -> ctypes.CDLL:
    """Load libfb.so (built in-tree by __graft_entry__.build()); raise if absent."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        raise RuntimeError(f"libfb.so not found at {path}: build it with "
                           "`python -m block_diffusion_attention_prefix_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in EXPORTED.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libfb takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libfb takes contiguous tensors (strides go through the shape)")
    return ctypes.c_void_p(t.data_ptr())


def _ptr_any(t: Optional[torch.Tensor]):
    """Device pointer of a tensor that may be a strided view (the strides go in the call)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libfb takes device tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(name: str, st: int):
    if st != 0:
        raise FBError(name, st, fb_status_string(st))


def make_shape(batch, h_q, h_kv, head_dim, block, n_prefix, dtype, kv_row_stride=0, kv_head_stride=0,
               scale=0.0) -> Shape:
    if isinstance(dtype, str):
        dtype = FB_F32 if dtype == "f32" else FB_BF16
    elif isinstance(dtype, torch.dtype):
        dtype = FB_F32 if dtype == torch.float32 else FB_BF16
    return Shape(batch, h_q, h_kv, head_dim, block, dtype, n_prefix, kv_row_stride, kv_head_stride, scale)


def make_gate(mask: torch.Tensor, first_step: bool, tau: int, head_sim: Optional[torch.Tensor] = None,
              gamma: float = 0.0) -> Gate:
    g = Gate(mask.data_ptr(), None if head_sim is None else head_sim.data_ptr(), int(bool(first_step)),
             int(tau), float(gamma))
    g._keep = (mask, head_sim)  # keep the tensors alive while the struct is in use
    return g


def _gref(g: Optional[Gate]):
    return None if g is None else ctypes.byref(g)


def fb_version() -> int:
    return load().fb_version()


def fb_status_string(st: int) -> str:
    return load().fb_status_string(st).decode()


def fb_device_error() -> int:
    code = ctypes.c_int32(0)
    _check("fb_device_error", load().fb_device_error(ctypes.byref(code)))
    return code.value


def fb_workspace_bytes(shape: Shape) -> int:
    return int(load().fb_workspace_bytes(ctypes.byref(shape)))


def fb_workspace_init(ws: torch.Tensor):
    _check("fb_workspace_init", load().fb_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream()))


def _wsargs(ws):
    return (_ptr(ws), 0 if ws is None else ws.numel() * ws.element_size())


def fb_gate_eval(shape, gate, dec_M, dec_reuse):
    _check("fb_gate_eval", load().fb_gate_eval(ctypes.byref(shape), _gref(gate), _ptr(dec_M), _ptr(dec_reuse),
                                               _stream()))


def fb_prefix_attn(shape, q, k_cache, v_cache, gate, a_out, l_out, ws):
    _check("fb_prefix_attn", load().fb_prefix_attn(
        ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), _gref(gate), _ptr(a_out), _ptr(l_out),
        *_wsargs(ws), _stream()))


def fb_block_attn(shape, q, k_blk, v_blk, a_in, l_in, ws=None):
    _check("fb_block_attn", load().fb_block_attn(
        ctypes.byref(shape), _ptr(q), _ptr(k_blk), _ptr(v_blk), _ptr(a_in), _ptr(l_in), *_wsargs(ws), _stream()))


def fb_merge(shape, a1, l1, a2, l2, a_full, l_full=None):
    _check("fb_merge", load().fb_merge(ctypes.byref(shape), _ptr(a1), _ptr(l1), _ptr(a2), _ptr(l2), _ptr(a_full),
                                       _ptr(l_full), _stream()))


def fb_merge_partials(shape, a_parts, a_part_stride, l_parts, l_part_stride, n_parts, gate, a_out, l_out):
    """Cache rows of recomputing heads = log-space merge of n_parts partials (strides in elements)."""
    _check("fb_merge_partials", load().fb_merge_partials(
        ctypes.byref(shape), _ptr_any(a_parts), int(a_part_stride), _ptr_any(l_parts), int(l_part_stride),
        int(n_parts), _gref(gate), _ptr(a_out), _ptr(l_out), _stream()))


def fb_exp2_fma(x: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = 2^x elementwise (float32, on the device) in the FMA-pipe arithmetic of the tcgen05 pass."""
    if x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 tensor")
    y = torch.empty_like(x) if y is None else y
    _check("fb_exp2_fma", load().fb_exp2_fma(_ptr(x), _ptr(y), x.numel(), _stream()))
    return y


def fb_block_merge(shape, q, k_blk, v_blk, gate, a_out, l_out, a_full, l_full=None, dec_M=None, dec_reuse=None,
                   ws=None):
    _check("fb_block_merge", load().fb_block_merge(
        ctypes.byref(shape), _ptr(q), _ptr(k_blk), _ptr(v_blk), _gref(gate), _ptr(a_out), _ptr(l_out),
        _ptr(a_full), _ptr(l_full), _ptr(dec_M), _ptr(dec_reuse), *_wsargs(ws), _stream()))


def fb_step(shape, q, k_cache, v_cache, k_blk, v_blk, gate, a_out, l_out, a_full, l_full, dec_M, dec_reuse, ws):
    _check("fb_step", load().fb_step(
        ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_blk), _ptr(v_blk), _gref(gate),
        _ptr(a_out), _ptr(l_out), _ptr(a_full), _ptr(l_full), _ptr(dec_M), _ptr(dec_reuse), *_wsargs(ws),
        _stream()))


def fb_prefix_attn_noalloc(shape, q, k_cache, v_cache, gate, a_out, l_out):
    """fb_prefix_attn with the workspace in library-owned static device memory (no allocation)."""
    _check("fb_prefix_attn_noalloc", load().fb_prefix_attn_noalloc(
        ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), _gref(gate), _ptr(a_out), _ptr(l_out),
        _stream()))


def fb_page_cap(shape, page_size=16) -> int:
    """Page stride of the [b, H_kv, D, page_cap] bounds layout for this shape."""
    n = int(load().fb_page_cap(ctypes.byref(shape), int(page_size)))
    if n <= 0:
        _check("fb_page_cap", n)
    return n


def fb_page_minmax(shape, k_cache, page_size, kmin, kmax):
    _check("fb_page_minmax", load().fb_page_minmax(ctypes.byref(shape), _ptr(k_cache), int(page_size), _ptr(kmin),
                                                   _ptr(kmax), _stream()))


def fb_append_block(shape, k_cache, v_cache, k_blk, v_blk, page_size=16, kmin=None, kmax=None):
    _check("fb_append_block", load().fb_append_block(ctypes.byref(shape), _ptr(k_cache), _ptr(v_cache), _ptr(k_blk),
                                                     _ptr(v_blk), int(page_size), _ptr(kmin), _ptr(kmax),
                                                     _stream()))


def fb_similarity_workspace_bytes(shape) -> int:
    return int(load().fb_similarity_workspace_bytes(ctypes.byref(shape)))


def fb_head_similarity(shape, q, q_ref, sim, ws):
    _check("fb_head_similarity", load().fb_head_similarity(ctypes.byref(shape), _ptr(q), _ptr(q_ref), _ptr(sim),
                                                           _ptr(ws), ws.numel() * ws.element_size(), _stream()))


def fb_refresh_reference(shape, q, q_ref, dec_reuse):
    _check("fb_refresh_reference", load().fb_refresh_reference(ctypes.byref(shape), _ptr(q), _ptr(q_ref),
                                                               _ptr(dec_reuse), _stream()))


def fb_losa_step(shape, q, q_prev, k_cache, v_cache, k_blk, v_blk, delta, sparse, a_full, l_full, mse, dec_active,
                 ws):
    _check("fb_losa_step", load().fb_losa_step(ctypes.byref(shape), _ptr(q), _ptr(q_prev), _ptr(k_cache),
                                               _ptr(v_cache), _ptr(k_blk), _ptr(v_blk), float(delta),
                                               ctypes.byref(sparse), _ptr(a_full), _ptr(l_full), _ptr(mse),
                                               _ptr(dec_active), _ptr(ws), ws.numel() * ws.element_size(),
                                               _stream()))


def fb_sparse_workspace_bytes(shape, page_size=16) -> int:
    return int(load().fb_sparse_workspace_bytes(ctypes.byref(shape), int(page_size)))


def fb_sparse_select(shape, q, gate, sparse, ws):
    _check("fb_sparse_select", load().fb_sparse_select(ctypes.byref(shape), _ptr(q), _gref(gate),
                                                       ctypes.byref(sparse), *_wsargs(ws), _stream()))


def fb_sparse_step(shape, q, k_cache, v_cache, k_blk, v_blk, gate, sparse, a_full, l_full, dec_M, dec_reuse, ws):
    _check("fb_sparse_step", load().fb_sparse_step(
        ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_blk), _ptr(v_blk), _gref(gate),
        ctypes.byref(sparse), _ptr(a_full), _ptr(l_full), _ptr(dec_M), _ptr(dec_reuse), *_wsargs(ws), _stream()))


class SparseResidualLayer:
    """Device buffers of one attention layer in sparse-residual mode, stepped through fb_sparse_step.

    Owns the page bounds (computed once from the prefix keys), the frozen selection,
    the residual cache, the outputs and the workspace.
    """

    def __init__(self, batch, h_q, h_kv, head_dim, block, k_cache, v_cache, n_select, page_size=16, scale=0.0,
                 keep_sel=False, n_prefix=None):
        # k_cache / v_cache [b, H_kv, capacity, D]; n_prefix (default: capacity) rows are the prefix.
        dev = k_cache.device
        cap = k_cache.shape[2]
        n = cap if n_prefix is None else int(n_prefix)
        self.shape = make_shape(batch, h_q, h_kv, head_dim, block, n, k_cache.dtype, scale=scale,
                                kv_head_stride=0 if n_prefix is None else cap * head_dim)
        self.k_cache, self.v_cache = k_cache, v_cache
        self.page_size = page_size
        self.n_pages = (n + page_size - 1) // page_size
        words = (self.n_pages + 31) // 32
        page_cap = fb_page_cap(self.shape, page_size)
        self.kmin = torch.empty((batch, h_kv, head_dim, page_cap), device=dev, dtype=k_cache.dtype)
        self.kmax = torch.empty_like(self.kmin)
        fb_page_minmax(self.shape, k_cache, page_size, self.kmin, self.kmax)
        i32, f32 = dict(device=dev, dtype=torch.int32), dict(device=dev, dtype=torch.float32)
        self.sel_idx = torch.zeros((batch, h_q, block, n_select), **i32)
        self.sel_bits = torch.zeros((batch, h_q, block, words), **i32)
        self.union_bits = torch.zeros((batch, h_kv, words), **i32)
        self.a_res = torch.zeros((batch, h_q, block, head_dim), **f32)
        self.l_res = torch.full((batch, h_q, block), float("-inf"), **f32)
        self.a_sel = torch.zeros((batch, h_q, block, head_dim), **f32) if keep_sel else None
        self.l_sel = torch.zeros((batch, h_q, block), **f32) if keep_sel else None
        self.a_full = torch.zeros((batch, h_q, block, head_dim), device=dev, dtype=k_cache.dtype)
        self.l_full = torch.zeros((batch, h_q, block), **f32)
        self.dec_M = torch.zeros((batch,), **i32)
        self.dec_reuse = torch.zeros((batch, h_q), device=dev, dtype=torch.uint8)
        nbytes = fb_sparse_workspace_bytes(self.shape, page_size)
        self.ws = torch.zeros(((nbytes + 15) // 16 * 16,), device=dev, dtype=torch.uint8)
        p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        self.sparse = Sparse(page_size, n_select, p(self.kmin), p(self.kmax), p(self.sel_idx), p(self.sel_bits),
                             p(self.union_bits), p(self.a_res), p(self.l_res), p(self.a_sel), p(self.l_sel))

    def step(self, q, k_blk, v_blk, mask, first_step, tau):
        g = make_gate(mask, first_step, tau)
        fb_sparse_step(self.shape, q, self.k_cache, self.v_cache, k_blk, v_blk, g, self.sparse, self.a_full,
                       self.l_full, self.dec_M, self.dec_reuse, self.ws)
        return self.a_full

    def finish_block(self, k_blk, v_blk, n_select):
        """Block transition: append the block's K/V to the prefix, refresh the page
        bounds it touched, and size the selection state for the grown prefix."""
        fb_append_block(self.shape, self.k_cache, self.v_cache, k_blk, v_blk, self.page_size, self.kmin, self.kmax)
        sh = self.shape
        self.shape = make_shape(sh.batch, sh.h_q, sh.h_kv, sh.head_dim, sh.block, sh.n_prefix + sh.block, sh.dtype,
                                kv_row_stride=sh.kv_row_stride, kv_head_stride=sh.kv_head_stride, scale=sh.scale)
        self.n_pages = (self.shape.n_prefix + self.page_size - 1) // self.page_size
        words = (self.n_pages + 31) // 32
        b, hq, B = sh.batch, sh.h_q, sh.block
        dev = self.k_cache.device
        self.sel_idx = torch.zeros((b, hq, B, n_select), device=dev, dtype=torch.int32)
        self.sel_bits = torch.zeros((b, hq, B, words), device=dev, dtype=torch.int32)
        self.union_bits = torch.zeros((b, sh.h_kv, words), device=dev, dtype=torch.int32)
        nbytes = fb_sparse_workspace_bytes(self.shape, self.page_size)
        self.ws = torch.zeros(((nbytes + 15) // 16 * 16,), device=dev, dtype=torch.uint8)
        sp = self.sparse
        self.sparse = Sparse(sp.page_size, n_select, sp.kmin, sp.kmax, self.sel_idx.data_ptr(),
                             self.sel_bits.data_ptr(), self.union_bits.data_ptr(), sp.a_res, sp.l_res, sp.a_sel,
                             sp.l_sel)


class CachedAttentionLayer:
    """Device buffers of one attention layer's FlashBlock state, stepped through fb_step.

    Owns (as torch tensors) the cache (A_out, L_out), the outputs (A_full, L_full),
    the decision record and the workspace.  The prefix K/V are the caller's.
    """

    def __init__(self, batch, h_q, h_kv, head_dim, block, k_cache: torch.Tensor, v_cache: torch.Tensor,
                 scale: float = 0.0, device=None, n_prefix=None):
        # k_cache / v_cache [b, H_kv, capacity, D]; n_prefix (default: capacity) rows are the prefix.
        dev = k_cache.device if device is None else device
        self.dtype = k_cache.dtype
        cap = k_cache.shape[2]
        self.shape = make_shape(batch, h_q, h_kv, head_dim, block, cap if n_prefix is None else int(n_prefix),
                                k_cache.dtype, scale=scale, kv_head_stride=0 if n_prefix is None else cap * head_dim)
        self.k_cache, self.v_cache = k_cache, v_cache
        f32 = dict(device=dev, dtype=torch.float32)
        self.a_out = torch.zeros((batch, h_q, block, head_dim), **f32)
        self.l_out = torch.full((batch, h_q, block), float("-inf"), **f32)
        self.a_full = torch.zeros((batch, h_q, block, head_dim), device=dev, dtype=self.dtype)
        self.l_full = torch.zeros((batch, h_q, block), **f32)
        self.dec_M = torch.zeros((batch,), device=dev, dtype=torch.int32)
        self.dec_reuse = torch.zeros((batch, h_q), device=dev, dtype=torch.uint8)
        nbytes = fb_workspace_bytes(self.shape)
        self.ws = torch.zeros(((nbytes + 15) // 16 * 16,), device=dev, dtype=torch.uint8)

    def step(self, q, k_blk, v_blk, mask, first_step, tau, head_sim=None, gamma=0.0):
        g = make_gate(mask, first_step, tau, head_sim, gamma)
        fb_step(self.shape, q, self.k_cache, self.v_cache, k_blk, v_blk, g, self.a_out, self.l_out,
                self.a_full, self.l_full, self.dec_M, self.dec_reuse, self.ws)
        return self.a_full

    def step_estimated(self, q, k_blk, v_blk, mask, first_step, tau, gamma):
        """A step whose per-head gamma gate uses the on-device similarity estimate:
        sim = cosine(q, the queries each head's cache was computed with); afterwards
        the recomputed heads' reference queries become q."""
        if not hasattr(self, "q_ref"):
            self.q_ref = torch.zeros_like(q)
            self.sim = torch.zeros((self.shape.batch, self.shape.h_q), device=q.device, dtype=torch.float32)
            n = fb_similarity_workspace_bytes(self.shape)
            self.sim_ws = torch.zeros(((n + 15) // 16 * 16,), device=q.device, dtype=torch.uint8)
        if not first_step:
            fb_head_similarity(self.shape, q, self.q_ref, self.sim, self.sim_ws)
        self.step(q, k_blk, v_blk, mask, first_step, tau, self.sim, gamma)
        fb_refresh_reference(self.shape, q, self.q_ref, self.dec_reuse)
        return self.a_full

    def finish_block(self, k_blk, v_blk):
        """Block transition: append the block's K/V to the prefix (the cache needs the
        capacity); the next block starts with first_step=True."""
        fb_append_block(self.shape, self.k_cache, self.v_cache, k_blk, v_blk)
        sh = self.shape
        self.shape = make_shape(sh.batch, sh.h_q, sh.h_kv, sh.head_dim, sh.block, sh.n_prefix + sh.block, sh.dtype,
                                kv_row_stride=sh.kv_row_stride, kv_head_stride=sh.kv_head_stride, scale=sh.scale)
        nbytes = fb_workspace_bytes(self.shape)
        if nbytes > self.ws.numel():
            self.ws = torch.zeros(((nbytes + 15) // 16 * 16,), device=self.ws.device, dtype=torch.uint8)


class LosaLayer(SparseResidualLayer):
    """One layer in LoSA mode: the first step of a block runs fb_step densely into the
    prefix cache (held in the sparse state's a_res / l_res); later steps run
    fb_losa_step with the previous step's queries."""

    def __init__(self, batch, h_q, h_kv, head_dim, block, k_cache, v_cache, n_select, delta, page_size=16,
                 scale=0.0, keep_sel=False):
        super().__init__(batch, h_q, h_kv, head_dim, block, k_cache, v_cache, n_select, page_size, scale, keep_sel)
        dev = k_cache.device
        self.delta = float(delta)
        self.mse = torch.zeros((batch, block), device=dev, dtype=torch.float32)
        self.active = torch.zeros((batch, block), device=dev, dtype=torch.uint8)
        nb = fb_workspace_bytes(self.shape)
        self.dense_ws = torch.zeros(((nb + 15) // 16 * 16,), device=dev, dtype=torch.uint8)
        self.q_prev = None

    def step(self, q, k_blk, v_blk, mask, first_step, tau=0):
        if first_step:
            g = make_gate(mask, True, 1)
            fb_step(self.shape, q, self.k_cache, self.v_cache, k_blk, v_blk, g, self.a_res, self.l_res,
                    self.a_full, self.l_full, self.dec_M, self.dec_reuse, self.dense_ws)
            self.active.fill_(1)
        else:
            fb_losa_step(self.shape, q, self.q_prev, self.k_cache, self.v_cache, k_blk, v_blk, self.delta,
                         self.sparse, self.a_full, self.l_full, self.mse, self.active, self.ws)
        self.q_prev = q.clone()
        return self.a_full
