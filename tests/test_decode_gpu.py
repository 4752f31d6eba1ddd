"""Token-level streaming decode through the C ABI: a sequence fed one token at a time
(pos = t mod N, fold on the last token) against the fp64 oracle's whole-sequence forward
(the oracle's decode step is pinned to that forward).  The segment of 1024 spreads a
token's keys over up to 16 ranges (CTAs) per (b, h), merged by a second launch.  Tolerances as for the forward:
bf16 max-abs 2e-2 / relative L2 5e-3 on the outputs, relative L2 5e-3 on the state;
fp32 max-abs 1e-4 and 1e-5."""

import numpy as np
import pytest
import torch

from compressive_memory_transformer_sm_b200 import DELTA, LINEAR, api
from compressive_memory_transformer_sm_b200 import workloads as W
from oracle import infini_ref as R

pytestmark = pytest.mark.gpu
DEV = "cuda"


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.mark.parametrize("mode", [LINEAR, DELTA], ids=["linear", "delta"])
@pytest.mark.parametrize("B,H,L,N,d,dtype", [(1, 2, 160, 64, 128, torch.bfloat16), (2, 1, 40, 16, 32, torch.float32),
                                             (1, 3, 130, 128, 128, torch.bfloat16),
                                             (1, 2, 1100, 1024, 128, torch.bfloat16)])
def test_decode_matches_forward(B, H, L, N, d, dtype, mode):
    w = W.Workload("decode", B=B, H=H, L=L, N=N, dk=d, dv=d, dtype=dtype, modes=(mode,), seed=4242 + L)
    q, k, v, beta = (t.to(DEV) for t in W.make_inputs(w, device="cpu"))
    M, z = torch.zeros(B, H, d, d, device=DEV), torch.zeros(B, H, d, device=DEV)
    kc = torch.zeros(B, H, N, d, dtype=dtype, device=DEV)
    vc = torch.zeros(B, H, N, d, dtype=dtype, device=DEV)
    out = torch.full((B, H, L, d), float("nan"), dtype=dtype, device=DEV)
    o_t = torch.empty(B, H, d, dtype=dtype, device=DEV)
    for t in range(L):
        api.infini_attn_decode_step(q[:, :, t].contiguous(), k[:, :, t].contiguous(), v[:, :, t].contiguous(),
                                    kc, vc, beta, M, z, o_t, t % N, mode, fold=(t == L - 1))
        out[:, :, t] = o_t
    torch.cuda.synchronize()
    assert api.infini_attn_device_status() == api.INFINI_OK
    wo, wM, wz = R.forward(np64(q), np64(k), np64(v), np64(beta), N, mode=mode)
    got = np64(out)
    assert np.all(np.isfinite(got))
    err, rl = float(np.max(np.abs(got - wo))), rel_l2(got, wo)
    if dtype == torch.float32:
        assert err <= 1e-4, f"out max-abs {err:.3e}"
        assert rel_l2(np64(M), wM) <= 1e-5 and rel_l2(np64(z), wz) <= 1e-5
    else:
        assert err <= 2e-2 and rl <= 5e-3, f"out max-abs {err:.3e} rel-L2 {rl:.3e}"
        assert rel_l2(np64(M), wM) <= 5e-3 and rel_l2(np64(z), wz) <= 5e-3
