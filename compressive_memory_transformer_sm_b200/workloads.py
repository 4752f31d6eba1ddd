"""Seeded synthetic workloads for the Infini-attention forward.

This module holds shapes and random-number recipes only -- none of the
method's arithmetic -- so that the CUDA path's tests and the CPU oracle can
be fed the same inputs without sharing any computation.

The shapes follow the explainer pages for arXiv 2404.07143 ("Leave No
Context Behind"): 8 heads of width 128 and segments of 2048 tokens for the
1B-scale language model (section 3, "Training infrastructure"), a 1M-token
passkey input processed segment by segment, and a 500K-token input for the
8B model; head count 32 and segment 8192 for the 8B shape are this
library's choice (the pages do not state them).  Every tensor is N(0, 1)
drawn in fp32 from ``torch.Generator(...).manual_seed(seed)`` and then cast
to the workload's dtype; beta is N(0, 1) per head; the memory starts empty.
"""

from __future__ import annotations

import dataclasses

import torch

LINEAR = 0
DELTA = 1
MODE_NAMES = {LINEAR: "linear", DELTA: "delta"}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    N: int
    dk: int
    dv: int
    dtype: torch.dtype
    modes: tuple
    seed: int
    streaming: bool = False

    @property
    def segments(self) -> int:
        return -(-self.L // self.N)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


TINY = Workload("tiny", B=1, H=2, L=32, N=8, dk=16, dv=16, dtype=torch.float32,
                modes=(LINEAR, DELTA), seed=1001)
LAYER_1B = Workload("1b_layer", B=1, H=8, L=32768, N=2048, dk=128, dv=128, dtype=torch.bfloat16,
                    modes=(LINEAR,), seed=1002)
BATCH_1B = Workload("1b_batch8", B=8, H=8, L=32768, N=2048, dk=128, dv=128, dtype=torch.bfloat16,
                    modes=(DELTA,), seed=1003)
PASSKEY_1M = Workload("passkey_1m_stream", B=1, H=8, L=1048576, N=2048, dk=128, dv=128,
                      dtype=torch.bfloat16, modes=(DELTA,), seed=1004, streaming=True)
LONG_8B = Workload("8b_long", B=2, H=32, L=524288, N=8192, dk=128, dv=128, dtype=torch.bfloat16,
                   modes=(LINEAR, DELTA), seed=1005)

WORKLOADS = {w.name: w for w in (TINY, LAYER_1B, BATCH_1B, PASSKEY_1M, LONG_8B)}


def make_inputs(w: Workload, device="cpu", seed=None):
    """q, k [B,H,L,dk], v [B,H,L,dv] in ``w.dtype`` and beta [H] fp32, all N(0, 1)."""
    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    q = torch.randn(w.B, w.H, w.L, w.dk, generator=g, device=device, dtype=torch.float32).to(w.dtype)
    k = torch.randn(w.B, w.H, w.L, w.dk, generator=g, device=device, dtype=torch.float32).to(w.dtype)
    v = torch.randn(w.B, w.H, w.L, w.dv, generator=g, device=device, dtype=torch.float32).to(w.dtype)
    beta = torch.randn(w.H, generator=g, device=device, dtype=torch.float32)
    return q, k, v, beta


def empty_state(w: Workload, device="cpu"):
    """M_0 = 0 [B,H,dk,dv] and z_0 = 0 [B,H,dk], fp32."""
    M = torch.zeros(w.B, w.H, w.dk, w.dv, device=device, dtype=torch.float32)
    z = torch.zeros(w.B, w.H, w.dk, device=device, dtype=torch.float32)
    return M, z


def random_state(w: Workload, device="cpu", seed=None, scale=1.0):
    """A non-empty starting memory with the shape the recurrence produces: z > 0.

    M_0 ~ scale * N(0, 1) and z_0 ~ scale * (1 + |N(0, 1)|) * tokens, where ``tokens``
    stands for the number of keys already written (N), so that the retrieval's
    denominator has the magnitude of a memory that has seen one segment.
    """
    g = torch.Generator(device=device)
    g.manual_seed((w.seed if seed is None else seed) + 7919)
    M = scale * torch.randn(w.B, w.H, w.dk, w.dv, generator=g, device=device) * (w.N ** 0.5)
    z = scale * (1.0 + torch.randn(w.B, w.H, w.dk, generator=g, device=device).abs()) * w.N
    return M.float(), z.float()


def make_layer_inputs(B: int, H: int, L: int, d_model: int, seed: int, device="cpu", head: int = 128):
    """Inputs of the full layer in bf16: x [B,L,D] ~ N(0, 1); w_qkv [D, 3*H*head] ~ N(0, 1/D)
    and w_o [H*head, D] ~ N(0, 1/(H*head)) (unit-variance projections); beta [H] fp32 ~ N(0, 1)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(B, L, d_model, generator=g, device=device).to(torch.bfloat16)
    w_qkv = (torch.randn(d_model, 3 * H * head, generator=g, device=device) / d_model ** 0.5).to(torch.bfloat16)
    w_o = (torch.randn(H * head, d_model, generator=g, device=device) / (H * head) ** 0.5).to(torch.bfloat16)
    beta = torch.randn(H, generator=g, device=device)
    return x, w_qkv, w_o, beta
