"""infini_attn_forward_noalloc against infini_attn_forward (collected last on purpose).

The no-allocation variant serves callers that may not allocate device memory
while they run (a serving loop that forbids allocation after start-up, a
fixed memory budget).  It takes its workspace from the library's fixed
32 MiB device buffer, so it must give exactly the results of the ordinary
call -- the kernels and their order of summation are the same, only the
workspace differs -- on consecutive calls that reuse the buffer, including
calls that find it dirty from a larger shape, and refuse shapes that need
more.
"""

import pytest
import torch

from compressive_memory_transformer_sm_b200 import DELTA, LINEAR, api
from compressive_memory_transformer_sm_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(seed, B=1, H=2, L=640):
    w = W.Workload("noalloc", B=B, H=H, L=L, N=1, dk=128, dv=128, dtype=torch.bfloat16, modes=(LINEAR,), seed=seed)
    return tuple(t.to(DEV) for t in W.make_inputs(w))


def _run(fn, q, k, v, beta, N, mode):
    B, H, L, d = q.shape
    M = torch.zeros(B, H, d, d, device=DEV)
    z = torch.zeros(B, H, d, device=DEV)
    out = torch.full_like(v, float("nan"))
    fn(q, k, v, beta, M, z, out, N, mode)
    torch.cuda.synchronize()
    assert api.infini_attn_device_status() == api.INFINI_OK
    return out, M, z


@pytest.mark.parametrize("mode", [DELTA, LINEAR])
def test_noalloc_matches_forward_on_two_calls_in_a_row(mode):
    N = 256
    # a larger call of the same rule first, so the checked calls find the
    # shared buffer full of another shape's snapshots and partials
    big = _inputs(30, H=8)
    assert api.infini_attn_workspace_size(1, 8, 640, N, 128, 128, mode) <= api.NOALLOC_SCRATCH_BYTES
    _run(api.infini_attn_forward_noalloc, *big, N, mode)
    q, k, v, beta = _inputs(31 + mode)
    B, H, L, d = q.shape
    want = _run(api.infini_attn_forward, q, k, v, beta, N, mode)
    for call in range(2):
        got = _run(api.infini_attn_forward_noalloc, q, k, v, beta, N, mode)
        for g, w_, name in zip(got, want, ("out", "M", "z")):
            assert torch.isfinite(g).all(), f"call {call} {name}: non-finite"
            assert torch.equal(g, w_), f"call {call} {name}: max-abs {(g.float() - w_.float()).abs().max().item():.3e}"


def test_noalloc_refuses_shapes_beyond_its_scratch():
    B, H, L, N = 1, 8, 32768, 2048
    assert api.infini_attn_workspace_size(B, H, L, N, 128, 128, LINEAR) > api.NOALLOC_SCRATCH_BYTES
    q = torch.empty(B, H, L, 128, dtype=torch.bfloat16, device=DEV)
    M = torch.zeros(B, H, 128, 128, device=DEV)
    z = torch.zeros(B, H, 128, device=DEV)
    beta = torch.zeros(H, device=DEV)
    out = torch.empty_like(q)
    rc = api.infini_attn_forward_noalloc(q, q, q, beta, M, z, out, N, LINEAR, raise_on_error=False)
    assert rc == api.INFINI_ERR_SCRATCH_LIMIT
    assert "32 MiB" in api.infini_attn_error_string(rc)
