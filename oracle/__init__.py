"""CPU oracle for the Infini-attention forward (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline
and reference arm may import this package.  The product path (the CUDA
library and its Python binding) never does.
"""

from . import brute, infini_ref  # noqa: F401
