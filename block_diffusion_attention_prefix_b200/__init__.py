"""Cached block-diffusion attention (FlashBlock) for B200 (sm_100a).

The compute path lives in ``libfb.so`` (hand-written CUDA behind a C-ABI declared
in ``include/fb.h``).  :mod:`.fb` is a thin ctypes binding with the same entry
point names; :mod:`.workloads` draws the seeded synthetic inputs.
"""
__all__ = ["fb", "workloads"]
