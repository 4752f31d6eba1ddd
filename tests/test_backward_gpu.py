"""Backward pass (back-propagation through time over the memory) through the C ABI, against
the fp64 oracle ``oracle.infini_bwd.backward`` (itself pinned to central finite differences
of the forward on the CPU).

The CUDA-core backward computes in fp32 from the inputs as given, so its error is fp32
rounding plus, for bf16 tensors, the final rounding of dq, dk, dv to bf16.  The tensor-core
path (bf16, head size 128) also rounds P and dS to bf16 as MMA operands and keeps A_dot in
bf16: each adds an independent relative error of about 2^-8 / sqrt(3) per element to sums of
mixed sign, about the size of the output rounding.  Tolerances (reasoned from that
arithmetic, the forward's in kind): fp32 tensors relative L2 1e-5 on every gradient; bf16
tensors relative L2 5e-3 on dq, dk, dv (output rounding alone gives about 1.7e-3, the
operand roundings of the tensor-core path about as much again) and 1e-4 on the fp32 outputs
dM0, dz0 (1e-3 on the tensor-core path).

dbeta = g (1 - g) sum dA . (A_mem - A_dot) is a sum of terms of both signs, so its error is
judged against the sum of their magnitudes, g (1 - g) sum |dA| (|A_mem| + |A_dot|) per head:
at most 1e-5 of it for fp32 tensors, 1e-4 for bf16 on CUDA cores, and 5e-3 on the tensor-core
path, whose recomputed A_dot carries the forward's bf16 rounding of P -- about 2^-9 relative
per element, not averaged away because V has random signs.
"""

import numpy as np
import pytest
import torch

from compressive_memory_transformer_sm_b200 import DELTA, LINEAR, api
from compressive_memory_transformer_sm_b200 import workloads as W
from oracle import infini_bwd as RB
from oracle import infini_ref as R
from tests.test_parity_gpu import DEV, inputs, np64, rel_l2

pytestmark = pytest.mark.gpu
NAMES = ("dq", "dk", "dv", "dbeta", "dM0", "dz0")


def _case(B, H, L, dk, dv, dtype, seed, state=False, final_grad=False):
    q, k, v, beta = inputs(B, H, L, dk, dv, dtype, seed)
    g = torch.Generator().manual_seed(seed + 1)
    d_out = torch.randn(B, H, L, dv, generator=g).to(dtype).to(DEV)
    M0 = z0 = dMS = dzS = None
    if state:
        w = W.Workload("s", B=B, H=H, L=L, N=8, dk=dk, dv=dv, dtype=dtype, modes=(LINEAR,), seed=seed)
        M0, z0 = (t.to(DEV) for t in W.random_state(w, scale=0.05))
    if final_grad:
        dMS = (0.01 * torch.randn(B, H, dk, dv, generator=g)).to(DEV)
        dzS = (0.001 * torch.randn(B, H, dk, generator=g)).to(DEV)
    return q, k, v, beta, d_out, M0, z0, dMS, dzS


def _compare(case, N, mode, f32, what, flags=0):
    q, k, v, beta, d_out, M0, z0, dMS, dzS = case
    tensor = not f32 and q.shape[3] == 128 and v.shape[3] == 128 and not (flags & api.FLAG_FORCE_SIMT)
    got = api.infini_attn_backward(q, k, v, beta, d_out, N, mode, M0=M0, z0=z0, dM_S=dMS, dz_S=dzS, flags=flags)
    torch.cuda.synchronize()
    assert api.infini_attn_device_status() == api.INFINI_OK
    n = lambda t: None if t is None else np64(t)  # noqa: E731
    want = RB.backward(np64(q), np64(k), np64(v), np64(beta), N, np64(d_out), n(dMS), n(dzS), mode=mode,
                       M0=n(M0), z0=n(z0))
    for name, gt, wt in zip(NAMES, got, want):
        gt = np64(gt)
        assert np.all(np.isfinite(gt)), f"{what} {name}: non-finite"
        if name == "dbeta":
            _, _, _, parts = R.forward(np64(q), np64(k), np64(v), np64(beta), N, mode=mode, M0=n(M0), z0=n(z0),
                                       return_parts=True)
            gw = 1.0 / (1.0 + np.exp(-np64(beta)))
            scale = gw * (1.0 - gw) * (np.abs(np64(d_out)) * (np.abs(parts["A_mem"]) + np.abs(parts["A_dot"]))).sum(
                axis=(0, 2, 3))
            rel = float(np.max(np.abs(gt - wt) / scale))
            tol = 1e-5 if f32 else (5e-3 if tensor else 1e-4)
            print(f"backward {what} dbeta: error / sum of |terms| {rel:.3e} (tolerance {tol:.0e})")
            assert rel <= tol, f"{what} dbeta: error {rel:.3e} of the sum of |terms| > {tol}"
            continue
        rl = rel_l2(gt, wt)
        tol = 1e-5 if f32 else (5e-3 if name in ("dq", "dk", "dv") else (1e-3 if tensor else 1e-4))
        print(f"backward {what} {name}: rel-L2 {rl:.3e} (tolerance {tol:.0e})")
        assert rl <= tol, f"{what} {name}: rel-L2 {rl:.3e} > {tol}"


@pytest.mark.parametrize("mode", [LINEAR, DELTA])
def test_backward_tiny_fp32(mode):
    w = W.TINY
    case = _case(w.B, w.H, w.L, w.dk, w.dv, torch.float32, w.seed)
    _compare(case, w.N, mode, True, f"tiny mode={mode}")


@pytest.mark.parametrize("shape", [(1, 2, 77, 10, 33, 7), (2, 1, 200, 32, 48, 64), (1, 2, 130, 128, 128, 40)])
@pytest.mark.parametrize("mode", [LINEAR, DELTA])
@pytest.mark.parametrize("extra", ["plain", "state+final"])
def test_backward_fp32_shapes(shape, mode, extra):
    B, H, L, dk, dv, N = shape
    case = _case(B, H, L, dk, dv, torch.float32, 50 + L + N, state=extra != "plain", final_grad=extra != "plain")
    _compare(case, N, mode, True, f"fp32 {shape} {extra} mode={mode}")


@pytest.mark.parametrize("shape", [(1, 2, 640, 256), (2, 1, 300, 128), (1, 1, 129, 129), (1, 2, 1000, 384)])
@pytest.mark.parametrize("mode", [LINEAR, DELTA])
@pytest.mark.parametrize("path", ["tensor", "simt"])
def test_backward_bf16(shape, mode, path):
    B, H, L, N = shape
    case = _case(B, H, L, 128, 128, torch.bfloat16, 70 + L + N, state=True, final_grad=True)
    _compare(case, N, mode, False, f"bf16 {path} {shape} mode={mode}",
             flags=api.FLAG_FORCE_SIMT if path == "simt" else 0)


@pytest.mark.parametrize("mode", [LINEAR, DELTA])
def test_backward_bf16_empty_state_long(mode):
    """Several full segments of 512 from the empty memory (zero retrieval rows in segment 1)."""
    case = _case(1, 2, 2048, 128, 128, torch.bfloat16, 81)
    _compare(case, 512, mode, False, f"bf16 tensor long mode={mode}")


@pytest.mark.parametrize("flags", [0, api.FLAG_FORCE_SIMT], ids=["tensor", "simt"])
def test_backward_deterministic_and_caller_workspace(flags):
    case = _case(1, 2, 384, 128, 128, torch.bfloat16, 91)
    q, k, v, beta, d_out = case[:5]
    a = api.infini_attn_backward(q, k, v, beta, d_out, 128, DELTA, flags=flags)
    ws = torch.empty(api.infini_attn_backward_workspace_size(1, 2, 384, 128, 128, 128, DELTA), dtype=torch.uint8,
                     device=DEV)
    b = api.infini_attn_backward(q, k, v, beta, d_out, 128, DELTA, workspace=ws, flags=flags)
    torch.cuda.synchronize()
    for x, y, name in zip(a, b, NAMES):
        assert torch.equal(x, y), name
