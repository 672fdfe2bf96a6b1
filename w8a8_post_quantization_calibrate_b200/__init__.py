"""SmoothQuant W8A8 smoothed linear layer on NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libsq.so`` (hand-written CUDA, declared
in ``include/sq.h``); ``sq`` is its thin ctypes binding and ``synth`` draws the
seeded synthetic workloads. Importing ``sq`` loads the library and raises if it
is missing: there is no CPU fallback.
"""
__all__ = ["sq", "synth"]
