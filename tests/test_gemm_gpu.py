"""The layer's projection GEMM (infini_attn_gemm_bf16, a tcgen05 kernel) against an fp64 product.

C = A B for bf16 A [M, K], B [K, N] with fp32 accumulation, rounded to bf16 (Eq. 5 and
Eq. 11 of the multi-head layer use it).  Every element must lie within bf16's unit
roundoff of the exact product -- 2^-8 relative: the 8-bit significand spaces values
2^(e-7) apart in [2^e, 2^(e+1)), so rounding to nearest moves a value by at most 2^(e-8),
up to 2^-8 of it -- plus the fp32 accumulation error, bounded by 2^-20 * sum_k |a_ik b_kj|.  Shapes cover several tiles, ragged M / N / K tails (N, K
multiples of 8), a single row, and the layer's shapes.
"""

import numpy as np
import pytest
import torch

from compressive_memory_transformer_sm_b200 import api

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(M, K, generator=g).to(torch.bfloat16)
    b = (torch.randn(K, N, generator=g) / K ** 0.5).to(torch.bfloat16)
    c = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    api.infini_attn_gemm_bf16(a.to(DEV), b.to(DEV), c)
    torch.cuda.synchronize()
    A, Bm = a.double().numpy(), b.double().numpy()
    ref = A @ Bm
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -20 * (np.abs(A) @ np.abs(Bm)) + 1e-30
    got = c.double().cpu().numpy()
    assert np.all(np.isfinite(got))
    excess = np.abs(got - ref) / bound
    assert float(excess.max()) <= 1.0, f"M={M} N={N} K={K}: worst element at {float(excess.max()):.3f} of its bound"


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (1, 8, 8), (300, 192, 200), (1000, 1032, 1032),
                                   (129, 520, 72), (2048, 768, 256)])
def test_gemm_shapes(M, N, K):
    _check(M, N, K, 1000 + M + N + K)


def test_gemm_layer_shapes():
    """The 1B-shaped layer's projections (d_model = 1024, H * 128 = 1024) on 4096 tokens."""
    _check(4096, 3 * 1024, 1024, 7)
    _check(4096, 1024, 1024, 8)


def test_gemm_rejects_unaligned_shapes():
    a = torch.zeros(16, 12, dtype=torch.bfloat16, device=DEV)
    b = torch.zeros(12, 16, dtype=torch.bfloat16, device=DEV)
    c = torch.zeros(16, 16, dtype=torch.bfloat16, device=DEV)
    assert api.infini_attn_gemm_bf16(a, b, c, raise_on_error=False) == api.INFINI_ERR_UNSUPPORTED
