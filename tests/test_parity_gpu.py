"""CUDA path (through the C ABI) against the fp64 oracle, element by element.

Tolerances: fp32 inputs max-abs 1e-4 on the output; bf16 inputs (fp32
accumulation) max-abs 2e-2 and relative L2 5e-3 on the output; the memory
state (M, z) within relative L2 5e-3 (bf16) or 1e-5 (fp32).  The oracle runs
in fp64 on the same bf16-rounded inputs.  The memory read A_mem is checked on
its own (gate forced to 1) because its magnitude, about 1/sqrt(tokens), hides
it under an absolute tolerance.
"""

import math

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


def assert_out(got, want, f32, what):
    err = float(np.max(np.abs(got - want))) if got.size else 0.0
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    if f32:
        assert err <= 1e-4, f"{what}: max-abs {err:.3e}"
    else:
        rl = rel_l2(got, want)
        assert err <= 2e-2 and rl <= 5e-3, f"{what}: max-abs {err:.3e} rel-L2 {rl:.3e}"


def assert_state(got, want, f32, what):
    rl = rel_l2(got, want)
    assert np.all(np.isfinite(got)), f"{what}: non-finite state"
    assert rl <= (1e-5 if f32 else 5e-3), f"{what}: rel-L2 {rl:.3e}"


def run(q, k, v, beta, N, mode, M0=None, z0=None, flags=0, use_ex=False, out=None):
    B, H, L, dk = q.shape
    dv = v.shape[3]
    M = torch.zeros(B, H, dk, dv, device=DEV) if M0 is None else M0.clone()
    z = torch.zeros(B, H, dk, device=DEV) if z0 is None else z0.clone()
    if out is None:
        out = torch.full((B, H, L, dv), float("nan"), dtype=q.dtype, device=DEV)
    if use_ex or flags:
        api.infini_attn_forward_ex(q, k, v, beta, M, z, out, N, mode, flags=flags)
    else:
        api.infini_attn_forward(q, k, v, beta, M, z, out, N, mode)
    torch.cuda.synchronize()
    assert api.infini_attn_device_status() == api.INFINI_OK
    return out, M, z


def inputs(B, H, L, dk, dv, dtype, seed):
    w = W.Workload("case", B=B, H=H, L=L, N=1, dk=dk, dv=dv, dtype=dtype, modes=(LINEAR,), seed=seed)
    q, k, v, beta = W.make_inputs(w, device="cpu")
    return q.to(DEV), k.to(DEV), v.to(DEV), beta.to(DEV)


def oracle(q, k, v, beta, N, mode, M0=None, z0=None, **kw):
    return R.forward(np64(q), np64(k), np64(v), np64(beta), N, mode=mode,
                     M0=None if M0 is None else np64(M0), z0=None if z0 is None else np64(z0), **kw)


def compare(q, k, v, beta, N, mode, f32, what, **kw):
    out, M, z = run(q, k, v, beta, N, mode, **kw)
    wo, wM, wz = oracle(q, k, v, beta, N, mode, kw.get("M0"), kw.get("z0"))
    assert_out(np64(out), wo, f32, what + " out")
    assert_state(np64(M), wM, f32, what + " M")
    assert_state(np64(z), wz, f32, what + " z")
    return out, M, z


# ----------------------------------------------------------------- fp32 path
@pytest.mark.parametrize("mode", [LINEAR, DELTA])
def test_tiny_fp32_workload(mode):
    w = W.TINY
    q, k, v, beta = (t.to(DEV) for t in W.make_inputs(w))
    compare(q, k, v, beta, w.N, mode, True, f"tiny mode={mode}")


@pytest.mark.parametrize("shape", [(1, 2, 77, 10, 33, 7), (2, 1, 200, 128, 128, 64), (1, 3, 65, 32, 48, 65),
                                   (1, 1, 1, 8, 8, 4)])
@pytest.mark.parametrize("mode", [LINEAR, DELTA])
def test_fp32_shapes(shape, mode):
    B, H, L, dk, dv, N = shape
    q, k, v, beta = inputs(B, H, L, dk, dv, torch.float32, 11 + L)
    compare(q, k, v, beta, N, mode, True, f"fp32 {shape} mode={mode}")


# ----------------------------------------------------------------- bf16 paths
BF16_SHAPES = [
    (1, 2, 1000, 384),  # 3 query tiles per segment, tail segment of 232
    (2, 1, 700, 200),   # segment length not a multiple of 128
    (1, 1, 300, 64),    # segment shorter than a tile
    (1, 3, 256, 256),   # exact tiles, two segments
    (1, 1, 129, 129),   # one token past a tile
]


PATH_FLAGS = {"tensor-pairs": api.FLAG_ATTN_PAIRS, "tensor-single": api.FLAG_ATTN_SINGLE,
              "tensor-split": api.FLAG_ATTN_SPLIT, "simt": api.FLAG_FORCE_SIMT}


@pytest.mark.parametrize("shape", BF16_SHAPES)
@pytest.mark.parametrize("mode", [LINEAR, DELTA])
@pytest.mark.parametrize("path", list(PATH_FLAGS))
def test_bf16_parity(shape, mode, path):
    B, H, L, N = shape
    q, k, v, beta = inputs(B, H, L, 128, 128, torch.bfloat16, 100 + L + N)
    compare(q, k, v, beta, N, mode, False, f"{path} {shape} mode={mode}", flags=PATH_FLAGS[path])


@pytest.mark.parametrize("mode", [LINEAR, DELTA])
@pytest.mark.parametrize("path", list(PATH_FLAGS))
def test_bf16_memory_read_alone(mode, path):
    """Gate forced to 1: out = A_mem, checked with the relative tolerance."""
    B, H, L, N = 1, 2, 1024, 256
    q, k, v, _ = inputs(B, H, L, 128, 128, torch.bfloat16, 7)
    beta = torch.full((H,), float("inf"), device=DEV)
    flags = PATH_FLAGS[path]
    out, _, _ = run(q, k, v, beta, N, mode, flags=flags)
    wo, _, _ = oracle(q, k, v, beta, N, mode)
    got = np64(out)
    assert np.all(got[:, :, :N] == 0.0), "empty memory must read zero in the first segment"
    assert rel_l2(got[:, :, N:], wo[:, :, N:]) <= 5e-3


@pytest.mark.parametrize("mode", [LINEAR, DELTA])
def test_bf16_local_attention_alone(mode):
    """Gate forced to 0: out = per-segment causal softmax attention."""
    B, H, L, N = 1, 2, 640, 256
    q, k, v, _ = inputs(B, H, L, 128, 128, torch.bfloat16, 8)
    beta = torch.full((H,), -float("inf"), device=DEV)
    out, _, _ = run(q, k, v, beta, N, mode)
    wo, _, _ = oracle(q, k, v, beta, N, mode)
    assert_out(np64(out), wo, False, "g=0")


@pytest.mark.parametrize("mode", [LINEAR, DELTA])
@pytest.mark.parametrize("path", list(PATH_FLAGS))
def test_bf16_nonempty_initial_state(mode, path):
    B, H, L, N = 2, 2, 512, 256
    q, k, v, beta = inputs(B, H, L, 128, 128, torch.bfloat16, 9)
    w = W.Workload("s", B=B, H=H, L=L, N=N, dk=128, dv=128, dtype=torch.bfloat16, modes=(mode,), seed=9)
    M0, z0 = (t.to(DEV) for t in W.random_state(w))
    flags = PATH_FLAGS[path]
    compare(q, k, v, beta, N, mode, False, f"{path} state0 mode={mode}", M0=M0, z0=z0, flags=flags)


@pytest.mark.parametrize("mode", [LINEAR, DELTA])
def test_bf16_strided_layout(mode):
    """[B, L, H, d] storage passed as strided [B, H, L, d] views through the extended call."""
    B, H, L, N = 2, 3, 520, 256
    g = torch.Generator().manual_seed(12)
    mk = lambda: torch.randn(B, L, H, 128, generator=g).to(torch.bfloat16).to(DEV)  # noqa: E731
    qs, ks, vs = mk(), mk(), mk()
    q, k, v = (t.permute(0, 2, 1, 3) for t in (qs, ks, vs))
    beta = torch.randn(H, generator=g).to(DEV)
    out_store = torch.full((B, L, H, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    out = out_store.permute(0, 2, 1, 3)
    o, M, z = run(q, k, v, beta, N, mode, use_ex=True, out=out)
    wo, wM, wz = oracle(q, k, v, beta, N, mode)
    assert_out(np64(o), wo, False, "strided out")
    assert_state(np64(M), wM, False, "strided M")


def test_explicit_scale_and_workspace():
    B, H, L, N = 1, 2, 384, 128
    q, k, v, beta = inputs(B, H, L, 128, 128, torch.bfloat16, 13)
    ws = torch.empty(api.infini_attn_workspace_size(B, H, L, N, 128, 128, DELTA), dtype=torch.uint8, device=DEV)
    M = torch.zeros(B, H, 128, 128, device=DEV)
    z = torch.zeros(B, H, 128, device=DEV)
    out = torch.empty_like(v)
    api.infini_attn_forward_ex(q, k, v, beta, M, z, out, N, DELTA, scale=0.2, workspace=ws)
    torch.cuda.synchronize()
    wo, wM, _ = oracle(q, k, v, beta, N, DELTA, scale=0.2)
    assert_out(np64(out), wo, False, "scale 0.2")
    assert_state(np64(M), wM, False, "scale 0.2 M")


def test_deterministic():
    B, H, L, N = 1, 2, 768, 256
    q, k, v, beta = inputs(B, H, L, 128, 128, torch.bfloat16, 14)
    for mode in (LINEAR, DELTA):
        a = run(q, k, v, beta, N, mode)
        b = run(q, k, v, beta, N, mode)
        for x, y in zip(a, b):
            assert torch.equal(x, y)


def test_bounded_wait_gives_up_and_context_survives():
    assert api.infini_attn_device_status(reset=True) == api.INFINI_OK
    assert api.infini_attn_selftest_timeout(2000) == api.INFINI_ERR_TIMEOUT
    assert api.infini_attn_device_status(reset=True) == api.INFINI_ERR_TIMEOUT
    assert api.infini_attn_device_status() == api.INFINI_OK
    q, k, v, beta = inputs(1, 1, 256, 128, 128, torch.bfloat16, 15)
    compare(q, k, v, beta, 128, DELTA, False, "after timeout self-test")


# ----------------------------------------------------------------- workloads at full size
def _sample_check_head(q, k, v, beta, out, M, z, b, h, N, mode, segments=None):
    """Oracle for one (b, h): the state trajectory in full, the output of sampled segments."""
    K, V, Q = np64(k[b, h]), np64(v[b, h]), np64(q[b, h])
    states, (Mf, zf) = R.memory_trajectory(K, V, N, mode)
    assert_state(np64(M[b, h]), Mf, False, f"M[{b},{h}]")
    assert_state(np64(z[b, h]), zf, False, f"z[{b},{h}]")
    bounds = R.segment_bounds(K.shape[0], N)
    segs = range(len(bounds)) if segments is None else segments
    got = np64(out[b, h])
    for si in segs:
        s0, s1 = bounds[si]
        want = R.segment_output(Q[s0:s1], K[s0:s1], V[s0:s1], *states[si], float(beta[h]))
        assert_out(got[s0:s1], want, False, f"out[{b},{h}] segment {si}")


def test_workload_1b_layer_linear():
    w = W.LAYER_1B
    q, k, v, beta = W.make_inputs(w, device=DEV)
    out, M, z = run(q, k, v, beta, w.N, LINEAR)
    for b, h in ((0, 0), (0, w.H - 1)):
        _sample_check_head(q, k, v, beta, out, M, z, b, h, w.N, LINEAR)
    # every head's final state against the closed form sum over all tokens
    K = np64(k[0])
    sk = np.where(K > 0, K + 1.0, np.exp(np.minimum(K, 0)))
    wantM = np.einsum("hti,htj->hij", sk, np64(v[0]))
    assert_state(np64(M[0]), wantM, False, "closed-form M")
    assert_state(np64(z[0]), sk.sum(axis=1), False, "closed-form z")


def test_workload_1b_batch8_delta():
    w = W.BATCH_1B
    q, k, v, beta = W.make_inputs(w, device=DEV)
    out, M, z = run(q, k, v, beta, w.N, DELTA)
    for b, h in ((0, 0), (w.B - 1, w.H - 1), (3, 5)):
        _sample_check_head(q, k, v, beta, out, M, z, b, h, w.N, DELTA, segments=[0, 1, 7, w.segments - 1])


def test_workload_passkey_1m_streaming_delta():
    """512 segment_step calls over 1M tokens: state stays [B,H,dk,dv] + [B,H,dk] fp32 and matches the oracle."""
    w = W.PASSKEY_1M
    q, k, v, beta = W.make_inputs(w, device=DEV)
    S = w.segments
    # the stream arrives one contiguous [B, H, N, d] segment at a time
    seg = lambda t: t.view(w.B, w.H, S, w.N, t.shape[3]).permute(2, 0, 1, 3, 4).contiguous()  # noqa: E731
    qs, ks, vs = seg(q), seg(k), seg(v)
    M, z = W.empty_state(w, device=DEV)
    outs = torch.empty_like(vs)
    state_bytes = M.numel() * 4 + z.numel() * 4
    assert state_bytes == 528384  # 8 x (128 x 128 + 128) x 4
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for s in range(S):
        api.infini_attn_segment_step(qs[s], ks[s], vs[s], beta, M, z, outs[s], DELTA)
    torch.cuda.synchronize()
    assert api.infini_attn_device_status() == api.INFINI_OK
    free1 = torch.cuda.mem_get_info()[0]
    assert abs(free1 - free0) < (64 << 20), "device memory grew across streaming steps"
    assert M.shape == (1, 8, 128, 128) and z.shape == (1, 8, 128)
    out = outs.permute(1, 2, 0, 3, 4).reshape(w.B, w.H, w.L, w.dv)
    _sample_check_head(q, k, v, beta, out, M, z, 0, 3, w.N, DELTA, segments=[0, 1, 2, 255, S - 1])


@pytest.mark.parametrize("shape", [(2, 3, 4 * 256 + 100, 256), (1, 2, 3 * 512, 512)])
@pytest.mark.parametrize("mode", [LINEAR, DELTA])
def test_segment_step_sequence_matches_forward(shape, mode):
    """One segment_step call per segment (ragged last segment in the first shape), bf16 d = 128 on
    the tensor cores (the update on the library's second stream, the attention on the caller's):
    outputs and final state equal the oracle's whole-sequence forward."""
    B, H, L, N = shape
    q, k, v, beta = inputs(B, H, L, 128, 128, torch.bfloat16, 300 + L + mode)
    M = torch.zeros(B, H, 128, 128, device=DEV)
    z = torch.zeros(B, H, 128, device=DEV)
    out = torch.full((B, H, L, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    for s0 in range(0, L, N):
        s1 = min(L, s0 + N)
        o = torch.empty(B, H, s1 - s0, 128, dtype=torch.bfloat16, device=DEV)
        api.infini_attn_segment_step(q[:, :, s0:s1].contiguous(), k[:, :, s0:s1].contiguous(),
                                     v[:, :, s0:s1].contiguous(), beta, M, z, o, mode)
        out[:, :, s0:s1] = o
    torch.cuda.synchronize()
    assert api.infini_attn_device_status() == api.INFINI_OK
    wo, wM, wz = oracle(q, k, v, beta, N, mode)
    what = f"segment_step {shape} mode={mode}"
    assert_out(np64(out), wo, False, what + " out")
    assert_state(np64(M), wM, False, what + " M")
    assert_state(np64(z), wz, False, what + " z")


def test_workload_8b_long_both_rules():
    w = W.LONG_8B
    q, k, v, beta = W.make_inputs(w, device=DEV)
    for mode in (LINEAR, DELTA):
        out, M, z = run(q, k, v, beta, w.N, mode)
        _sample_check_head(q, k, v, beta, out, M, z, w.B - 1, w.H - 1, w.N, mode, segments=[0, 1, w.segments - 1])
        del out


# ----------------------------------------------------------------- memory read alone, full size
def _check_amem_head(q, k, v, out, b, h, N, mode, segments, what):
    """Gate forced to 1 (out = A_mem): relative L2 of sampled segments against the oracle's
    sigma(Q) M_{s-1} / (sigma(Q) z_{s-1}), with M_{s-1}, z_{s-1} from the oracle's own trajectory."""
    K, V, Q = np64(k[b, h]), np64(v[b, h]), np64(q[b, h])
    states, _ = R.memory_trajectory(K, V, N, mode)
    bounds = R.segment_bounds(K.shape[0], N)
    got = np64(out[b, h])
    worst = 0.0
    for si in segments:
        s0, s1 = bounds[si]
        want = R.memory_retrieval(R.elu_plus_one(Q[s0:s1]), *states[si])
        rl = rel_l2(got[s0:s1], want)
        print(f"A_mem alone {what} (b={b}, h={h}) segment {si}: rel-L2 {rl:.3e} "
              f"(tolerance 5e-3, margin {5e-3 / rl:.1f}x)")
        assert np.all(np.isfinite(got[s0:s1]))
        assert rl <= 5e-3, f"A_mem {what} segment {si}: rel-L2 {rl:.3e}"
        worst = max(worst, rl)
    return worst


def test_memory_read_alone_full_size():
    """A_mem at full size on every workload (both rules on the 8B shape): its magnitude,
    about 1/sqrt(tokens), would hide under the output's absolute tolerance, so the gate is
    forced to 1 and the relative tolerance applies to A_mem itself."""
    cases = [(W.LONG_8B, LINEAR, [(W.LONG_8B.B - 1, W.LONG_8B.H - 1)], [1, 2, 63]),
             (W.LONG_8B, DELTA, [(W.LONG_8B.B - 1, W.LONG_8B.H - 1)], [1, 2, 63]),
             (W.BATCH_1B, DELTA, [(0, 0), (7, 7)], [1, 7, 15])]
    for w, mode, heads, segs in cases:
        q, k, v, _ = W.make_inputs(w, device=DEV)
        beta = torch.full((w.H,), float("inf"), device=DEV)
        out, _, _ = run(q, k, v, beta, w.N, mode)
        for b, h in heads:
            _check_amem_head(q, k, v, out, b, h, w.N, mode, segs, f"{w.name} mode={mode}")
        del q, k, v, out
        torch.cuda.empty_cache()
    # the passkey stream, one segment_step call per segment
    w = W.PASSKEY_1M
    q, k, v, _ = W.make_inputs(w, device=DEV)
    beta = torch.full((w.H,), float("inf"), device=DEV)
    S = w.segments
    seg = lambda t: t.view(w.B, w.H, S, w.N, t.shape[3]).permute(2, 0, 1, 3, 4).contiguous()  # noqa: E731
    qs, ks, vs = seg(q), seg(k), seg(v)
    M, z = W.empty_state(w, device=DEV)
    outs = torch.empty_like(vs)
    for s in range(S):
        api.infini_attn_segment_step(qs[s], ks[s], vs[s], beta, M, z, outs[s], DELTA)
    torch.cuda.synchronize()
    assert api.infini_attn_device_status() == api.INFINI_OK
    out = outs.permute(1, 2, 0, 3, 4).reshape(w.B, w.H, w.L, w.dv)
    _check_amem_head(q, k, v, out, 0, 3, w.N, DELTA, [1, 255, S - 1], "passkey_1m_stream")
