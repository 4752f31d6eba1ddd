"""Infini-attention forward for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libinfini_attn.so`` (hand-written
CUDA kernels); ``api`` is its thin ctypes binding and ``workloads`` holds the
seeded synthetic inputs.  Importing the binding loads the library and raises
if it has not been built -- there is no CPU fallback.
"""

LINEAR = 0
DELTA = 1
F32 = 0x10

__all__ = ["LINEAR", "DELTA", "F32"]
