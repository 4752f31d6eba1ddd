"""infini_attn_forward_noalloc against infini_attn_forward (collected last on purpose).

The no-allocation variant serves callers that may not allocate device memory
while they run (a serving loop that forbids allocation after start-up, a
fixed memory budget).  It takes its workspace from the library's fixed
32 MiB device buffer, so it must give the same results as the ordinary call,
on consecutive calls that reuse the buffer, and refuse shapes that need more.
"""

import numpy as np
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
    return [t.double().cpu().numpy() for t in (out, M, z)]


def _close(a, b, what):
    err = float(np.max(np.abs(a - b)))
    rel = float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
    assert np.all(np.isfinite(a)), what
    assert err <= 2e-2 and rel <= 5e-3, f"{what}: max-abs {err:.3e} rel-L2 {rel:.3e}"


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    N = 256
    for call, (seed, mode) in enumerate(((31, DELTA), (32, LINEAR))):
        q, k, v, beta = _inputs(seed)
        B, H, L, d = q.shape
        assert api.infini_attn_workspace_size(B, H, L, N, d, d, mode) <= api.NOALLOC_SCRATCH_BYTES
        got = _run(api.infini_attn_forward_noalloc, q, k, v, beta, N, mode)
        want = _run(api.infini_attn_forward, q, k, v, beta, N, mode)
        for g, w_, name in zip(got, want, ("out", "M", "z")):
            _close(g, w_, f"call {call} {name}")


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
