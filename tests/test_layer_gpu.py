"""Full layer (projections + Infini-attention + output projection) through the C ABI
against the fp64 oracle's ``layer_forward`` on the same bf16 inputs.

The oracle keeps Q, K, V and the concatenated head outputs in bf16 between its
steps, as the library does (see the oracle's header); tolerances as for the bf16
attention: max-abs 2e-2 and relative L2 5e-3 on the output, relative L2 5e-3 on
the memory state.
"""

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
@pytest.mark.parametrize("B,H,L,N,D", [(1, 2, 640, 256, 256), (2, 1, 300, 128, 192), (1, 3, 384, 384, 384)])
@pytest.mark.parametrize("nonempty", [False, True], ids=["empty", "state"])
def test_layer_parity(B, H, L, N, D, mode, nonempty):
    x, w_qkv, w_o, beta = (t.to(DEV) for t in W.make_layer_inputs(B, H, L, D, seed=9000 + B * 100 + H * 10 + L))
    if nonempty:
        M0, z0 = W.random_state(W.Workload("s", B=B, H=H, L=L, N=N, dk=128, dv=128, dtype=torch.bfloat16,
                                           modes=(mode,), seed=77), device=DEV)
    else:
        M0, z0 = torch.zeros(B, H, 128, 128, device=DEV), torch.zeros(B, H, 128, device=DEV)
    M, z = M0.clone(), z0.clone()
    y = torch.full((B, L, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    api.infini_attn_layer_forward(x, w_qkv, w_o, beta, M, z, y, H, N, mode)
    torch.cuda.synchronize()
    assert api.infini_attn_device_status() == api.INFINI_OK
    wy, wM, wz = R.layer_forward(np64(x), np64(w_qkv), np64(w_o), np64(beta), H, N, mode=mode,
                                 M0=np64(M0), z0=np64(z0))
    got = np64(y)
    assert np.all(np.isfinite(got))
    err, rl = float(np.max(np.abs(got - wy))), rel_l2(got, wy)
    assert err <= 2e-2 and rl <= 5e-3, f"y: max-abs {err:.3e} rel-L2 {rl:.3e}"
    assert rel_l2(np64(M), wM) <= 5e-3 and rel_l2(np64(z), wz) <= 5e-3


def test_layer_caller_workspace_matches_own():
    B, H, L, N, D = 1, 2, 512, 256, 256
    x, w_qkv, w_o, beta = (t.to(DEV) for t in W.make_layer_inputs(B, H, L, D, seed=9100))
    ys = []
    for use_ws in (False, True):
        M, z = torch.zeros(B, H, 128, 128, device=DEV), torch.zeros(B, H, 128, device=DEV)
        y = torch.empty(B, L, D, dtype=torch.bfloat16, device=DEV)
        ws = None
        if use_ws:
            ws = torch.empty(api.infini_attn_layer_workspace_size(B, H, L, N, D, DELTA), dtype=torch.uint8, device=DEV)
        api.infini_attn_layer_forward(x, w_qkv, w_o, beta, M, z, y, H, N, DELTA, workspace=ws)
        torch.cuda.synchronize()
        ys.append((y.clone(), M.clone(), z.clone()))
    for a, b in zip(ys[0], ys[1]):
        assert torch.equal(a, b)
