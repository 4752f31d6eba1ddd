"""Rotary position embeddings on the local attention only, through the C ABI, against the oracle.

Section 4.1 of the paper (quoted on the explainer page "Leave No Context Behind"): the
dot-product attention's Q and K carry position embeddings, the compressive memory's do not.
The oracle's ``forward(..., rope_base=...)`` rotates Q, K for A_dot only (pinned on the CPU:
rotation = complex multiplication, state and memory read unchanged, output invariant to a
shift of every position).  Here the CUDA path must match it at the workloads' tolerances.
"""

import numpy as np
import pytest
import torch

from compressive_memory_transformer_sm_b200 import DELTA, LINEAR, api
from compressive_memory_transformer_sm_b200 import workloads as W
from oracle import infini_ref as R
from tests.test_parity_gpu import (BF16_SHAPES, DEV, PATH_FLAGS, assert_out, assert_state, inputs, np64)

pytestmark = pytest.mark.gpu
BASE = 10000.0


def run_rope(q, k, v, beta, N, mode, base=BASE, offset=0, flags=0, out=None, M0=None, z0=None, workspace=None):
    B, H, L, dk = q.shape
    dv = v.shape[3]
    M = torch.zeros(B, H, dk, dv, device=DEV) if M0 is None else M0.clone()
    z = torch.zeros(B, H, dk, device=DEV) if z0 is None else z0.clone()
    if out is None:
        out = torch.full((B, H, L, dv), float("nan"), dtype=q.dtype, device=DEV)
    api.infini_attn_forward_ex(q, k, v, beta, M, z, out, N, mode, flags=flags, rope_base=base, rope_offset=offset,
                               workspace=workspace)
    torch.cuda.synchronize()
    assert api.infini_attn_device_status() == api.INFINI_OK
    return out, M, z


def oracle_rope(q, k, v, beta, N, mode, base=BASE, offset=0, M0=None, z0=None):
    return R.forward(np64(q), np64(k), np64(v), np64(beta), N, mode=mode, rope_base=base, rope_offset=offset,
                     M0=None if M0 is None else np64(M0), z0=None if z0 is None else np64(z0))


def compare_rope(q, k, v, beta, N, mode, f32, what, **kw):
    oracle_kw = {x: kw[x] for x in ("base", "offset", "M0", "z0") if x in kw}
    out, M, z = run_rope(q, k, v, beta, N, mode, **kw)
    wo, wM, wz = oracle_rope(q, k, v, beta, N, mode, **oracle_kw)
    assert_out(np64(out), wo, f32, what + " out")
    assert_state(np64(M), wM, f32, what + " M")
    assert_state(np64(z), wz, f32, what + " z")
    return out


@pytest.mark.parametrize("shape", BF16_SHAPES)
@pytest.mark.parametrize("mode", [LINEAR, DELTA])
@pytest.mark.parametrize("path", list(PATH_FLAGS))
def test_rope_bf16_parity(shape, mode, path):
    B, H, L, N = shape
    q, k, v, beta = inputs(B, H, L, 128, 128, torch.bfloat16, 300 + L + N)
    compare_rope(q, k, v, beta, N, mode, False, f"rope {path} {shape} mode={mode}", flags=PATH_FLAGS[path])


@pytest.mark.parametrize("shape", [(1, 2, 77, 10, 33, 7), (1, 3, 65, 32, 48, 65), (2, 1, 200, 128, 128, 64)])
@pytest.mark.parametrize("mode", [LINEAR, DELTA])
def test_rope_fp32_parity(shape, mode):
    B, H, L, dk, dv, N = shape
    q, k, v, beta = inputs(B, H, L, dk, dv, torch.float32, 400 + L)
    compare_rope(q, k, v, beta, N, mode, True, f"rope fp32 {shape} mode={mode}")


@pytest.mark.parametrize("offset", [37, 500_000, 2_000_000_000])
def test_rope_position_offset(offset):
    """Large positions: the angle is reduced modulo 2 pi in fp64 before the fp32 sine and cosine."""
    q, k, v, beta = inputs(1, 2, 640, 128, 128, torch.bfloat16, 17)
    compare_rope(q, k, v, beta, 256, DELTA, False, f"rope offset {offset}", offset=offset)


def test_rope_changes_only_the_local_branch():
    """Same state as without position embeddings (bit for bit), the memory read unchanged
    (gate forced to 1), and a different output where the local branch counts."""
    q, k, v, beta = inputs(1, 2, 768, 128, 128, torch.bfloat16, 18)
    for mode in (LINEAR, DELTA):
        o0, M0, z0 = run_rope(q, k, v, beta, 256, mode, base=0.0)
        o1, M1, z1 = run_rope(q, k, v, beta, 256, mode)
        assert torch.equal(M0, M1) and torch.equal(z0, z1)
        assert not torch.equal(o0, o1)
        inf = torch.full_like(beta, float("inf"))
        a0, _, _ = run_rope(q, k, v, inf, 256, mode, base=0.0)
        a1, _, _ = run_rope(q, k, v, inf, 256, mode)
        assert torch.equal(a0, a1)


def test_rope_strided_layout_state_and_workspace():
    """[B, L, H, d] storage as strided views, a non-empty initial state and a caller workspace
    sized by infini_attn_workspace_size_ex."""
    B, H, L, N = 2, 3, 520, 256
    g = torch.Generator().manual_seed(19)
    mk = lambda: torch.randn(B, L, H, 128, generator=g).to(torch.bfloat16).to(DEV)  # noqa: E731
    q, k, v = (t.permute(0, 2, 1, 3) for t in (mk(), mk(), mk()))
    beta = torch.randn(H, generator=g).to(DEV)
    w = W.Workload("s", B=B, H=H, L=L, N=N, dk=128, dv=128, dtype=torch.bfloat16, modes=(DELTA,), seed=19)
    M0, z0 = (t.to(DEV) for t in W.random_state(w))
    nbytes = api.infini_attn_workspace_size_ex(B, H, L, N, 128, 128, DELTA, rope_base=BASE)
    assert nbytes > api.infini_attn_workspace_size(B, H, L, N, 128, 128, DELTA)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    out = torch.full((B, L, H, 128), float("nan"), dtype=torch.bfloat16, device=DEV).permute(0, 2, 1, 3)
    compare_rope(q, k, v, beta, N, DELTA, False, "rope strided", out=out, M0=M0, z0=z0, workspace=ws)


def test_rope_workload_1b_layer_sampled_heads():
    """The 1B-shaped layer with position embeddings: state trajectory in full for two heads and
    the output of sampled segments against the oracle's segment recurrence with rotated Q, K."""
    w = W.LAYER_1B
    q, k, v, beta = W.make_inputs(w, device=DEV)
    out, M, z = run_rope(q, k, v, beta, w.N, LINEAR)
    for b, h in ((0, 0), (0, w.H - 1)):
        Q, K, V = np64(q[b, h]), np64(k[b, h]), np64(v[b, h])
        states, (Mf, zf) = R.memory_trajectory(K, V, w.N, LINEAR)
        assert_state(np64(M[b, h]), Mf, False, f"M[{b},{h}]")
        assert_state(np64(z[b, h]), zf, False, f"z[{b},{h}]")
        bounds = R.segment_bounds(w.L, w.N)
        got = np64(out[b, h])
        for si in (0, 1, 7, w.segments - 1):
            s0, s1 = bounds[si]
            pos = np.arange(s0, s1, dtype=np.float64)
            want, _, _, _ = R.infini_attention_segment(Q[s0:s1], K[s0:s1], V[s0:s1], *states[si], float(beta[h]),
                                                       LINEAR, q_local=R.rope(Q[s0:s1], pos, BASE),
                                                       k_local=R.rope(K[s0:s1], pos, BASE))
            assert_out(got[s0:s1], want, False, f"rope 1b out[{b},{h}] segment {si}")
