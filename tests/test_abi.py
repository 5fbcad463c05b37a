"""C-ABI checks that need no GPU: the library loads, exports every symbol that
include/fb.h declares, its structs have the binding's layout, and host-side
validation rejects bad arguments with a status before any launch."""
import ctypes
import os
import re
import subprocess

import pytest

from block_diffusion_attention_prefix_b200 import fb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fb.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fb_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(fb.lib_path()):
        from block_diffusion_attention_prefix_b200 import build
        build.build()
    return fb.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("fb_prefix_attn", "fb_block_attn", "fb_merge", "fb_step"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(fb.EXPORTED), "binding misses a declared entry point"


def test_struct_layout_matches_c(tmp_path, lib):
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "fb.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu %zu %zu\\n\", sizeof(fb_shape), offsetof(fb_shape, n_prefix),"
        " offsetof(fb_shape, scale), sizeof(fb_gate), offsetof(fb_gate, tau), offsetof(fb_gate, gamma));return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = list(map(int, subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()))
    want = [ctypes.sizeof(fb.Shape), fb.Shape.n_prefix.offset, fb.Shape.scale.offset, ctypes.sizeof(fb.Gate),
            fb.Gate.tau.offset, fb.Gate.gamma.offset]
    assert got == want


def test_status_strings(lib):
    assert fb.fb_version() >= 100
    for st in range(0, -9, -1):
        assert lib.fb_status_string(st)
    assert lib.fb_status_string(-8) != lib.fb_status_string(-1)


def S(**kw):
    base = dict(batch=1, h_q=4, h_kv=2, head_dim=128, block=4, n_prefix=256, dtype=fb.FB_BF16)
    base.update(kw)
    return fb.make_shape(**base)


ALIGNED = ctypes.c_void_p(0x10000)       # never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10008)


def call_prefix(lib, shape, q=ALIGNED, k=ALIGNED, v=ALIGNED, a=ALIGNED, l=ALIGNED, gate=None, ws=ALIGNED,
                ws_bytes=1 << 30):
    return lib.fb_prefix_attn(None if shape is None else ctypes.byref(shape), q, k, v,
                              None if gate is None else ctypes.byref(gate), a, l, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dtype=7), -4),
    (dict(batch=0), -2),
    (dict(h_q=6, h_kv=4), -2),
    (dict(block=0), -2),
    (dict(n_prefix=-1), -2),
    (dict(head_dim=96), -7),               # bf16 supports D = 64, 128
    (dict(head_dim=256, dtype=fb.FB_F32), -7),
    (dict(kv_row_stride=100), -2),         # smaller than head_dim
    (dict(kv_row_stride=132), -3),         # 264 bytes: not a multiple of 16
    (dict(scale=float("nan")), -8),
    (dict(scale=-1.0), -8),
])
def test_bad_shapes_are_rejected_before_launch(lib, kw, status):
    assert call_prefix(lib, S(**kw)) == status


def test_null_and_misaligned_pointers(lib):
    assert call_prefix(lib, None) == -1
    assert call_prefix(lib, S(), q=None) == -1
    assert call_prefix(lib, S(), a=MISALIGNED) == -3
    assert call_prefix(lib, S(), k=MISALIGNED) == -3
    assert call_prefix(lib, S(), ws=None) == -5
    assert call_prefix(lib, S(), ws=MISALIGNED) == -3
    g = fb.Gate(None, None, 0, 2, 0.0)
    assert call_prefix(lib, S(), gate=g) == -1          # gate without its mask
    g = fb.Gate(0x10000, 0x10004, 0, 2, 0.5)
    assert call_prefix(lib, S(), gate=g) == -3          # misaligned head_sim


def test_step_requires_gate_and_workspace(lib):
    sh = S()
    args = [ALIGNED] * 5
    st = lib.fb_step(ctypes.byref(sh), *args, None, *[ALIGNED] * 6, ALIGNED, 1 << 30, None)
    assert st == -1
    assert lib.fb_merge(ctypes.byref(sh), ALIGNED, None, ALIGNED, ALIGNED, ALIGNED, None, None) == -1


def test_workspace_bytes_for_valid_and_invalid_shapes(lib):
    assert fb.fb_workspace_bytes(S(dtype=9)) == 0
    n = fb.fb_workspace_bytes(S())
    assert n > 0 and n % 4 == 0
    big = fb.fb_workspace_bytes(S(n_prefix=800_000, h_q=32, h_kv=8))
    assert big >= n


@pytest.mark.parametrize("n,cap,want", [   # ceil(capacity / 16) rounded up to a multiple of 8
    (1, None, 8), (16, None, 8), (17, None, 8), (65536, None, 4096), (65536, 65552, 4104), (1000, 2000, 128),
    (2000, None, 128), (2048, None, 128), (2049, None, 136),
])
def test_page_cap_is_the_pages_of_the_cache_capacity(lib, n, cap, want):
    kw = dict(n_prefix=n) if cap is None else dict(n_prefix=n, kv_head_stride=cap * 128)
    assert fb.fb_page_cap(S(**kw)) == want


def test_page_cap_rejects_other_page_sizes(lib):
    assert lib.fb_page_cap(ctypes.byref(S()), 8) == -8      # FB_ERR_ARG
    assert lib.fb_page_cap(ctypes.byref(S(n_prefix=0)), 16) == -7  # FB_ERR_UNSUPPORTED


def test_sparse_and_similarity_workspace_queries(lib):
    sh = S(h_q=32, h_kv=8, n_prefix=65536)
    n = fb.fb_sparse_workspace_bytes(sh, 16)
    assert (1 << 20) < n < (64 << 20)                      # partials, in-block slot, f64 estimates
    assert fb.fb_sparse_workspace_bytes(S(h_q=32, h_kv=8, n_prefix=2 * 65536), 16) > n   # estimates grow with N
    assert fb.fb_sparse_workspace_bytes(sh, 8) == 0         # page size 16 only
    assert fb.fb_sparse_workspace_bytes(S(dtype=9), 16) == 0
    assert fb.fb_similarity_workspace_bytes(S(h_q=12, h_kv=12, block=4680)) > 0
    assert fb.fb_similarity_workspace_bytes(S(batch=0)) == 0
