"""Pins that tie the fp64 oracle to what the pages and the mathematics fix.

Each ``pin_*`` function takes the oracle module (``oracle.infini_ref`` or a
deliberately broken copy of it) and returns a list of failure messages
(empty when the pin holds).  ``test_oracle.py`` runs them against the real
oracle; ``test_oracle_mutations.py`` plants plausible mistakes in the oracle
and checks that at least one pin catches each.

Sources, all on the explainer page "Leave No Context Behind: Efficient
Infinite Context Transformers with Infini-attention" (section 3, Technical
Approach) unless stated: Eq. 6 (local causal attention), Eq. 7 (retrieval),
the closed forms of M_{s-1} and z_{s-1}, Eq. 8 / Eq. 9 (updates), Eq. 10
(gate), Eq. 4 (recurrent contract), the delta rule's "binding already
exists" property (also on the paperlayer.ai summary, section 3), and the
per-layer footprint of d_key x d_value + d_key per head.
"""

from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import torch

from oracle import brute

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _expr(s: str) -> float:
    """Evaluate a golden-file input expression built from numbers, ln(), sqrt() and unary minus."""
    return float(eval(s, {"__builtins__": {}}, {"ln": math.log, "sqrt": math.sqrt}))


def _frac(s: str) -> float:
    return float(Fraction(s))


def _rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (scale * torch.randn(*shape, generator=g, dtype=torch.float64)).numpy()


def _close(a, b, tol, what):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    if a.shape != b.shape:
        return [f"{what}: shape {a.shape} vs {b.shape}"]
    if not np.all(np.isfinite(a)):
        return [f"{what}: non-finite values"]
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    return [] if err <= tol else [f"{what}: max abs err {err:.3e} > {tol:.1e}"]


# ---------------------------------------------------------------------------
def pin_hand_examples(ref):
    """Hand-derived worked examples (tests/golden/hand_examples.json)."""
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        data = json.load(f)
    fails = []
    for ex in data["examples"]:
        q = np.array([[_expr(x) for x in row] for row in ex["q"]])[None, None]
        k = np.array([[_expr(x) for x in row] for row in ex["k"]])[None, None]
        v = np.array([[_expr(x) for x in row] for row in ex["v"]])[None, None]
        beta = np.array([_expr(ex["beta"])])
        want_out = np.array([[_frac(x) for x in row] for row in ex["out"]])
        for mode, key in ((ref.LINEAR, "linear"), (ref.DELTA, "delta")):
            out, M, z = ref.forward(q, k, v, beta, ex["N"], mode=mode)
            fails += _close(out[0, 0], want_out, 1e-12, f"{ex['name']}/{key} out")
            fails += _close(M[0, 0], np.array([[_frac(x) for x in r] for r in ex[key]["M"]]), 1e-12,
                            f"{ex['name']}/{key} M")
            fails += _close(z[0, 0], np.array([_frac(x) for x in ex[key]["z"]]), 1e-12, f"{ex['name']}/{key} z")
    return fails


def pin_sigma(ref):
    """sigma = ELU + 1 (alpha = 1): identity + 1 above 0, exp at and below 0, continuous, positive."""
    x = np.array([-30.0, -2.0, -math.log(2.0), -1e-9, 0.0, 1e-9, 0.5, 3.0])
    want = np.array([math.exp(-30.0), math.exp(-2.0), 0.5, math.exp(-1e-9), 1.0, 1.0 + 1e-9, 1.5, 4.0])
    fails = _close(ref.elu_plus_one(x), want, 1e-15, "sigma values")
    if not np.all(ref.elu_plus_one(np.linspace(-50, 50, 1001)) > 0):
        fails.append("sigma not positive")
    return fails


def pin_gate_zero_is_sdpa(ref):
    """beta -> -inf gives g = 0: out equals per-segment causal softmax attention
    computed by torch's scaled_dot_product_attention in float64 (Eq. 6, Eq. 10)."""
    fails = []
    B, H, L, dk, dv = 2, 3, 23, 8, 5
    q, k, v = _rand((B, H, L, dk), 1), _rand((B, H, L, dk), 2), _rand((B, H, L, dv), 3)
    beta = np.full(H, -np.inf)
    for N in (L, 7, 4, 1):
        scale = 1.0 / math.sqrt(dk)
        out, _, _ = ref.forward(q, k, v, beta, N, mode=ref.LINEAR)
        want = np.zeros_like(out)
        for s0 in range(0, L, N):
            s1 = min(L, s0 + N)
            want[:, :, s0:s1] = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[:, :, s0:s1]), torch.from_numpy(k[:, :, s0:s1]),
                torch.from_numpy(v[:, :, s0:s1]), is_causal=True, scale=scale).numpy()
        fails += _close(out, want, 1e-12, f"g=0 vs SDPA (N={N})")
        out_d, _, _ = ref.forward(q, k, v, beta, N, mode=ref.DELTA)
        fails += _close(out_d, want, 1e-12, f"g=0 delta vs SDPA (N={N})")
    return fails


def pin_linear_closed_form(ref):
    """Linear rule: M_S = sum_t sigma(k_t)^T v_t and z_S = sum_t sigma(k_t) over every token,
    hence independent of the segment length N (closed forms under Eq. 7)."""
    fails = []
    B, H, L, dk, dv = 1, 2, 24, 6, 4
    q, k, v = _rand((B, H, L, dk), 4), _rand((B, H, L, dk), 5), _rand((B, H, L, dv), 6)
    beta = _rand((H,), 7)
    sk = np.where(k > 0, k + 1.0, np.exp(np.minimum(k, 0)))  # ELU + 1, written out independently
    want_M = np.einsum("bhti,bhtj->bhij", sk, v)
    want_z = sk.sum(axis=2)
    for N in (24, 12, 6, 5, 1):
        _, M, z = ref.forward(q, k, v, beta, N, mode=ref.LINEAR)
        fails += _close(M, want_M, 1e-11, f"linear M closed form (N={N})")
        fails += _close(z, want_z, 1e-11, f"linear z closed form (N={N})")
    return fails


def pin_brute_linear(ref):
    """Segmentwise oracle == token-by-token normalised linear attention over earlier segments."""
    fails = []
    B, H, L, dk, dv = 1, 2, 13, 3, 2
    q, k, v = _rand((B, H, L, dk), 8), _rand((B, H, L, dk), 9), _rand((B, H, L, dv), 10)
    beta = _rand((H,), 11)
    for N in (4, 5):
        out, M, z = ref.forward(q, k, v, beta, N, mode=ref.LINEAR)
        bo, bM, bz = brute.forward_linear_closed_form(q.tolist(), k.tolist(), v.tolist(), beta.tolist(), N)
        fails += _close(out, np.array(bo), 1e-12, f"brute linear out (N={N})")
        fails += _close(M, np.array(bM), 1e-12, f"brute linear M (N={N})")
        fails += _close(z, np.array(bz), 1e-12, f"brute linear z (N={N})")
    # memory read alone: beta -> +inf makes out = A_mem
    big = np.full(H, np.inf)
    out, _, _ = ref.forward(q, k, v, big, 4, mode=ref.LINEAR)
    bo, _, _ = brute.forward_linear_closed_form(q.tolist(), k.tolist(), v.tolist(), big.tolist(), 4)
    fails += _close(out, np.array(bo), 1e-12, "brute A_mem (g=1)")
    return fails


def pin_brute_delta(ref):
    """Segmentwise oracle == element-loop evaluation of the delta rule on tiny inputs."""
    fails = []
    B, H, L, dk, dv = 1, 2, 11, 3, 2
    q, k, v = _rand((B, H, L, dk), 12), _rand((B, H, L, dk), 13), _rand((B, H, L, dv), 14)
    beta = _rand((H,), 15)
    for N in (3, 4, 11):
        out, M, z = ref.forward(q, k, v, beta, N, mode=ref.DELTA)
        bo, bM, bz = brute.forward_delta_loops(q.tolist(), k.tolist(), v.tolist(), beta.tolist(), N)
        fails += _close(out, np.array(bo), 1e-12, f"brute delta out (N={N})")
        fails += _close(M, np.array(bM), 1e-12, f"brute delta M (N={N})")
        fails += _close(z, np.array(bz), 1e-12, f"brute delta z (N={N})")
    return fails


def pin_delta_fixed_point(ref):
    """Delta rule leaves M unchanged when V already equals what the memory returns for K,
    while z still grows by sum_t sigma(K_t)."""
    fails = []
    dk, dv, n = 5, 4, 9
    M0 = _rand((dk, dv), 16)
    z0 = np.abs(_rand((dk,), 17)) + 3.0
    Ks = _rand((n, dk), 18)
    sk = np.where(Ks > 0, Ks + 1.0, np.exp(np.minimum(Ks, 0)))
    Vs = (sk @ M0) / (sk @ z0)[:, None]
    M1, z1 = ref.delta_update(M0, z0, ref.elu_plus_one(Ks), Vs)
    fails += _close(M1, M0, 1e-12, "delta fixed point M")
    fails += _close(z1, z0 + sk.sum(axis=0), 1e-12, "delta fixed point z")
    # and through the full segment recurrence with a non-empty starting memory
    q = _rand((1, 1, n, dk), 19)
    _, M2, z2 = ref.forward(q, Ks[None, None], Vs[None, None], np.zeros(1), n, mode=ref.DELTA,
                            M0=M0[None, None], z0=z0[None, None])
    fails += _close(M2[0, 0], M0, 1e-12, "delta fixed point via forward M")
    fails += _close(z2[0, 0], z0 + sk.sum(axis=0), 1e-12, "delta fixed point via forward z")
    return fails


def pin_delta_first_segment(ref):
    """From empty memory, one segment of the delta rule equals the linear rule: M = sigma(K)^T V."""
    fails = []
    n, dk, dv = 7, 4, 3
    q, k, v = _rand((1, 1, n, dk), 20), _rand((1, 1, n, dk), 21), _rand((1, 1, n, dv), 22)
    sk = np.where(k > 0, k + 1.0, np.exp(np.minimum(k, 0)))[0, 0]
    for mode in (ref.LINEAR, ref.DELTA):
        _, M, z = ref.forward(q, k, v, np.zeros(1), n, mode=mode)
        fails += _close(M[0, 0], sk.T @ v[0, 0], 1e-12, f"first segment M (mode {mode})")
        fails += _close(z[0, 0], sk.sum(axis=0), 1e-12, f"first segment z (mode {mode})")
    return fails


def pin_gate_extremes(ref):
    """g = 1 gives pure memory (0 in the first segment); g = 1/2 averages A_mem and A_dot (Eq. 10)."""
    fails = []
    B, H, L, dk, dv, N = 1, 2, 12, 4, 4, 4
    q, k, v = _rand((B, H, L, dk), 23), _rand((B, H, L, dk), 24), _rand((B, H, L, dv), 25)
    for mode in (ref.LINEAR, ref.DELTA):
        out1, _, _ = ref.forward(q, k, v, np.full(H, np.inf), N, mode=mode)
        out0, _, _ = ref.forward(q, k, v, np.full(H, -np.inf), N, mode=mode)
        outh, _, _ = ref.forward(q, k, v, np.zeros(H), N, mode=mode)
        fails += _close(out1[:, :, :N], np.zeros((B, H, N, dv)), 0.0, "g=1 first segment")
        fails += _close(outh, 0.5 * (out0 + out1), 1e-12, "g=1/2 average")
        if np.max(np.abs(out1[:, :, N:])) == 0.0:
            fails.append("g=1 later segments are all zero")
    return fails


def pin_streaming_resume(ref):
    """Eq. 4 contract: forward(L) == S single-segment steps == forward(L1) then forward(L - L1)."""
    fails = []
    B, H, L, dk, dv, N = 2, 2, 20, 4, 3, 5
    q, k, v = _rand((B, H, L, dk), 26), _rand((B, H, L, dk), 27), _rand((B, H, L, dv), 28)
    beta = _rand((H,), 29)
    for mode in (ref.LINEAR, ref.DELTA):
        out, M, z = ref.forward(q, k, v, beta, N, mode=mode)
        Ms, zs = np.zeros((B, H, dk, dv)), np.zeros((B, H, dk))
        outs = []
        for s0 in range(0, L, N):
            o, Ms, zs = ref.segment_step(q[:, :, s0:s0 + N], k[:, :, s0:s0 + N], v[:, :, s0:s0 + N], beta, Ms, zs,
                                         mode=mode)
            outs.append(o)
        fails += _close(np.concatenate(outs, axis=2), out, 1e-12, f"streaming out (mode {mode})")
        fails += _close(Ms, M, 1e-12, f"streaming M (mode {mode})")
        L1 = 10
        o1, M1, z1 = ref.forward(q[:, :, :L1], k[:, :, :L1], v[:, :, :L1], beta, N, mode=mode)
        o2, M2, z2 = ref.forward(q[:, :, L1:], k[:, :, L1:], v[:, :, L1:], beta, N, mode=mode, M0=M1, z0=z1)
        fails += _close(np.concatenate([o1, o2], axis=2), out, 1e-12, f"resume out (mode {mode})")
        fails += _close(M2, M, 1e-12, f"resume M (mode {mode})")
        fails += _close(z2, z, 1e-12, f"resume z (mode {mode})")
    return fails


def pin_head_permutation(ref):
    """Heads are independent (multi-head section, Eq. 11): permuting heads permutes outputs and state."""
    B, H, L, dk, dv, N = 1, 4, 9, 3, 3, 4
    q, k, v = _rand((B, H, L, dk), 30), _rand((B, H, L, dk), 31), _rand((B, H, L, dv), 32)
    beta = _rand((H,), 33)
    perm = np.array([2, 0, 3, 1])
    fails = []
    for mode in (ref.LINEAR, ref.DELTA):
        out, M, z = ref.forward(q, k, v, beta, N, mode=mode)
        po, pM, pz = ref.forward(q[:, perm], k[:, perm], v[:, perm], beta[perm], N, mode=mode)
        fails += _close(po, out[:, perm], 1e-13, f"permuted heads (mode {mode})")
        fails += _close(pM, M[:, perm], 1e-13, f"permuted heads M (mode {mode})")
    return fails


def pin_state_size(ref):
    """Memory of H (d_key d_value + d_key) numbers per layer, independent of L; the page's figures."""
    with open(os.path.join(GOLDEN, "memory_footprint.json")) as f:
        g = json.load(f)
    fails = []
    n = ref.state_numbers(g["H"], g["dk"], g["dv"])
    if n != g["matrix_numbers_per_layer"] + g["normaliser_numbers_per_layer"]:
        fails.append(f"state numbers {n}")
    total = n * g["layers"] / 1e6
    if abs(total - g["total_memory_parameters_millions_approx"]) > 0.05:
        fails.append(f"12-layer total {total}M")
    if abs(n * 4 / 2**20 - g["fp32_bytes_per_layer_approx_MB"]) > 0.01:
        fails.append("fp32 bytes per layer")
    ratio = g["memorizing_transformer_memory_parameters_millions"] / g["total_memory_parameters_millions_approx"]
    if round(ratio) != g["compression_vs_memorizing_transformer_approx"]:
        fails.append(f"compression ratio {ratio}")
    if len(ref.segment_bounds(g["training_length"], g["segment_length"])) != g["segments_per_training_sequence"]:
        fails.append("segments per training sequence")
    # state shapes after forwards of different lengths
    for L in (4, 17, 40):
        q = _rand((1, 2, L, 3), 34)
        _, M, z = ref.forward(q, q, q[..., :2], np.zeros(2), 4, mode=ref.DELTA)
        if M.shape != (1, 2, 3, 2) or z.shape != (1, 2, 3):
            fails.append(f"state shape depends on L={L}")
    return fails


def pin_tail_segment(ref):
    """A short last segment is causal inside itself and updates M, z over its own tokens only."""
    fails = []
    B, H, L, dk, dv, N = 1, 1, 11, 3, 2, 4
    q, k, v = _rand((B, H, L, dk), 35), _rand((B, H, L, dk), 36), _rand((B, H, L, dv), 37)
    beta = _rand((H,), 38)
    for mode in (ref.LINEAR, ref.DELTA):
        out, M, z = ref.forward(q, k, v, beta, N, mode=mode)
        o8, M8, z8 = ref.forward(q[:, :, :8], k[:, :, :8], v[:, :, :8], beta, N, mode=mode)
        ot, Mt, zt = ref.segment_step(q[:, :, 8:], k[:, :, 8:], v[:, :, 8:], beta, M8, z8, mode=mode)
        fails += _close(np.concatenate([o8, ot], axis=2), out, 1e-12, f"tail segment out (mode {mode})")
        fails += _close(Mt, M, 1e-12, f"tail segment M (mode {mode})")
    return fails


def pin_flop_count(ref):
    """Algorithmic FLOPs: 2(dk+dv) per unmasked (query, key) pair plus 2 dk dv per token for each
    memory product (2 products for linear, 3 for delta), counted by brute force over the mask."""
    fails = []
    for (B, H, L, N, dk, dv) in ((1, 2, 10, 4, 3, 5), (2, 1, 9, 9, 2, 2)):
        for mode, prods in ((ref.LINEAR, 2), (ref.DELTA, 3)):
            pairs = 0
            for s0 in range(0, L, N):
                n = min(N, L - s0)
                pairs += sum(1 for i in range(n) for j in range(n) if j <= i)
            want = B * H * (pairs * 2 * (dk + dv) + L * prods * 2 * dk * dv)
            got = ref.forward_flops(B, H, L, N, dk, dv, mode)
            if got != want:
                fails.append(f"flops {got} != {want}")
    return fails


ALL_PINS = [
    pin_hand_examples, pin_sigma, pin_gate_zero_is_sdpa, pin_linear_closed_form, pin_brute_linear,
    pin_brute_delta, pin_delta_fixed_point, pin_delta_first_segment, pin_gate_extremes,
    pin_streaming_resume, pin_head_permutation, pin_state_size, pin_tail_segment, pin_flop_count,
]


def run_all(ref):
    """Run every pin; returns {pin name: [failures]} for the pins that failed or raised."""
    bad = {}
    for pin in ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                f = pin(ref)
        except Exception as e:  # a broken oracle may raise instead of returning wrong numbers
            f = [f"raised {type(e).__name__}: {e}"]
        if f:
            bad[pin.__name__] = f
    return bad


def pin_trajectory(ref):
    """The update-only trajectory and per-segment outputs reproduce the full forward."""
    fails = []
    L, dk, dv, N = 19, 4, 3, 5
    q, k, v = _rand((1, 1, L, dk), 40), _rand((1, 1, L, dk), 41), _rand((1, 1, L, dv), 42)
    beta = _rand((1,), 43)
    for mode in (ref.LINEAR, ref.DELTA):
        out, M, z = ref.forward(q, k, v, beta, N, mode=mode)
        states, (Mf, zf) = ref.memory_trajectory(k[0, 0], v[0, 0], N, mode)
        fails += _close(Mf, M[0, 0], 1e-12, f"trajectory M (mode {mode})")
        fails += _close(zf, z[0, 0], 1e-12, f"trajectory z (mode {mode})")
        for si, (s0, s1) in enumerate(ref.segment_bounds(L, N)):
            A = ref.segment_output(q[0, 0, s0:s1], k[0, 0, s0:s1], v[0, 0, s0:s1], *states[si], beta[0])
            fails += _close(A, out[0, 0, s0:s1], 1e-12, f"segment output {si} (mode {mode})")
    return fails


ALL_PINS.append(pin_trajectory)


# ---------------------------------------------------------------------------
def pin_layer_identity(ref):
    """With W_Q = W_K = W_V = I and W_O = I (d_model = H d) the layer reduces to the
    recurrence on X split into heads (Eq. 5 and Eq. 11 with identity projections)."""
    fails = []
    B, H, L, dk, N = 2, 3, 11, 4, 4
    D = H * dk
    x = _rand((B, L, D), 50)
    beta = _rand((H,), 51)
    eye = np.eye(D)
    w_qkv = np.concatenate([eye, eye, eye], axis=1)
    xh = x.reshape(B, L, H, dk).transpose(0, 2, 1, 3)
    for mode in (ref.LINEAR, ref.DELTA):
        y, M, z = ref.layer_forward(x, w_qkv, eye, beta, H, N, mode=mode, dk=dk, round_intermediates=False)
        out, M2, z2 = ref.forward(xh, xh, xh, beta, N, mode=mode)
        fails += _close(y, out.transpose(0, 2, 1, 3).reshape(B, L, D), 1e-12, f"identity layer output (mode {mode})")
        fails += _close(M, M2, 1e-12, f"identity layer M (mode {mode})")
        fails += _close(z, z2, 1e-12, f"identity layer z (mode {mode})")
    return fails


ALL_PINS.append(pin_layer_identity)


def pin_layer_loops(ref):
    """Projections written out as sums over the model dimension, element by element
    (Eq. 5: q_j = sum_c x_c W_Q[c, j]; Eq. 11: o_c = sum_{h, j} a_{h, j} W_O[h d + j, c]),
    around the recurrence, on a tiny layer with d_model != H d."""
    fails = []
    B, H, L, dk, N, D = 1, 2, 5, 3, 2, 4
    x = _rand((B, L, D), 60)
    w_qkv = _rand((D, 3 * H * dk), 61, 0.5)
    w_o = _rand((H * dk, D), 62, 0.5)
    beta = _rand((H,), 63)
    proj = np.zeros((3, B, H, L, dk))
    for blk in range(3):
        for b in range(B):
            for h in range(H):
                for t in range(L):
                    for j in range(dk):
                        proj[blk, b, h, t, j] = sum(x[b, t, c] * w_qkv[c, blk * H * dk + h * dk + j] for c in range(D))
    for mode in (ref.LINEAR, ref.DELTA):
        out, _, _ = ref.forward(proj[0], proj[1], proj[2], beta, N, mode=mode)
        want = np.zeros((B, L, D))
        for b in range(B):
            for t in range(L):
                for c in range(D):
                    want[b, t, c] = sum(out[b, h, t, j] * w_o[h * dk + j, c] for h in range(H) for j in range(dk))
        y, _, _ = ref.layer_forward(x, w_qkv, w_o, beta, H, N, mode=mode, dk=dk, round_intermediates=False)
        fails += _close(y, want, 1e-12, f"layer vs element-wise projections (mode {mode})")
    return fails


ALL_PINS.append(pin_layer_loops)


def pin_bf16_rounding(ref):
    """The layer's bf16 storage equals torch's round-to-nearest-even bfloat16 cast."""
    a = _rand((4096,), 70, 3.0)
    a[:4] = [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 2.0 ** -130]  # ties and a denormal
    want = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    got = ref.bf16_round(a)
    return [] if np.array_equal(got, want) else ["bf16_round differs from torch's bfloat16 cast"]


ALL_PINS.append(pin_bf16_rounding)


def pin_decode_matches_forward(ref):
    """Token-by-token decode (a cache per segment, folded into the memory when the
    segment completes, and at the last token) reproduces the whole-sequence forward:
    outputs and final state, both rules, with a short tail segment."""
    fails = []
    B, H, L, dk, dv, N = 2, 2, 13, 3, 4, 5
    q, k, v = _rand((B, H, L, dk), 80), _rand((B, H, L, dk), 81), _rand((B, H, L, dv), 82)
    beta = _rand((H,), 83)
    for mode in (ref.LINEAR, ref.DELTA):
        want, wM, wz = ref.forward(q, k, v, beta, N, mode=mode)
        M, z = np.zeros((B, H, dk, dv)), np.zeros((B, H, dk))
        kc, vc = np.zeros((B, H, N, dk)), np.zeros((B, H, N, dv))
        got = np.zeros_like(want)
        for t in range(L):
            got[:, :, t], M, z = ref.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], kc, vc, beta, M, z, t % N,
                                                 mode=mode, fold=(t == L - 1))
        fails += _close(got, want, 1e-12, f"decode outputs (mode {mode})")
        fails += _close(M, wM, 1e-12, f"decode final M (mode {mode})")
        fails += _close(z, wz, 1e-12, f"decode final z (mode {mode})")
    return fails


ALL_PINS.append(pin_decode_matches_forward)


# ---------------------------------------------------------------------------
def pin_rope_as_complex_rotation(ref):
    """The rotary embedding equals multiplying each pair (x_2i + i x_2i+1) by exp(i p base^(-2i/d))."""
    n, d, base = 7, 8, 10000.0
    x = _rand((n, d), 90)
    pos = np.array([0, 1, 2, 5, 11, 100, 2047], dtype=np.float64)
    zc = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * pos[:, None] * base ** (-np.arange(0, d, 2) / d)[None, :])
    want = np.empty_like(x)
    want[:, 0::2], want[:, 1::2] = zc.real, zc.imag
    fails = _close(ref.rope(x, pos, base), want, 1e-12, "rope vs complex rotation")
    fails += _close(ref.rope(x, np.zeros(n), base), x, 0.0, "rope at position 0")
    return fails


ALL_PINS.append(pin_rope_as_complex_rotation)


def pin_rope_split(ref):
    """Position embeddings on the local branch only (section 4.1): the memory state and the
    memory read are those of the forward without them; the local branch alone is causal
    softmax attention on the rotated Q, K (torch SDPA, per segment); and it depends only on
    relative positions, so shifting every position leaves the output unchanged."""
    fails = []
    B, H, L, d, N, base = 1, 2, 23, 6, 8, 500.0
    q, k, v = _rand((B, H, L, d), 91), _rand((B, H, L, d), 92), _rand((B, H, L, d), 93)
    beta = _rand((H,), 94)
    for mode in (ref.LINEAR, ref.DELTA):
        o0, M0, z0 = ref.forward(q, k, v, beta, N, mode=mode)
        o1, M1, z1 = ref.forward(q, k, v, beta, N, mode=mode, rope_base=base)
        fails += _close(M1, M0, 1e-12, f"rope leaves M unchanged (mode {mode})")
        fails += _close(z1, z0, 1e-12, f"rope leaves z unchanged (mode {mode})")
        inf = np.full(H, np.inf)
        fails += _close(ref.forward(q, k, v, inf, N, mode=mode, rope_base=base)[0],
                        ref.forward(q, k, v, inf, N, mode=mode)[0], 1e-12, f"memory read without PE (mode {mode})")
        shifted = ref.forward(q, k, v, beta, N, mode=mode, rope_base=base, rope_offset=37)[0]
        fails += _close(shifted, o1, 1e-9, f"rope output shift-invariant (mode {mode})")
    # local branch alone against SDPA on rotated Q, K computed with complex numbers
    ninf = np.full(H, -np.inf)
    got = ref.forward(q, k, v, ninf, N, rope_base=base)[0]
    want = np.zeros_like(got)
    for s0 in range(0, L, N):
        s1 = min(L, s0 + N)
        pos = np.arange(s0, s1, dtype=np.float64)
        rot = np.exp(1j * pos[:, None] * base ** (-np.arange(0, d, 2) / d)[None, :])

        def rc(t):
            zc = (t[..., 0::2] + 1j * t[..., 1::2]) * rot
            out = np.empty_like(t)
            out[..., 0::2], out[..., 1::2] = zc.real, zc.imag
            return out

        qs, ks = rc(q[:, :, s0:s1]), rc(k[:, :, s0:s1])
        want[:, :, s0:s1] = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qs), torch.from_numpy(ks), torch.from_numpy(v[:, :, s0:s1]), is_causal=True).numpy()
    fails += _close(got, want, 1e-12, "local branch with rope vs SDPA")
    return fails


ALL_PINS.append(pin_rope_split)


# ---------------------------------------------------------------------------
def pin_backward_finite_differences(ref):
    """The back-propagation oracle (``oracle.infini_bwd``) against central finite
    differences of the forward, every coordinate of q, k, v, beta, M_0, z_0, both rules,
    three segments with a tail, a non-empty initial memory (z_0 > 0)."""
    from oracle import infini_bwd

    fails = []
    B, H, L, dk, dv, N = 1, 2, 7, 3, 2, 3
    q, k, v = _rand((B, H, L, dk), 100), _rand((B, H, L, dk), 101), _rand((B, H, L, dv), 102)
    beta = _rand((H,), 103)
    M0 = _rand((B, H, dk, dv), 104)
    z0 = 1.0 + np.abs(_rand((B, H, dk), 105))
    W_out, W_M, w_z = _rand((B, H, L, dv), 106), _rand((B, H, dk, dv), 107), _rand((B, H, dk), 108)
    for mode in (ref.LINEAR, ref.DELTA):
        def loss(q_, k_, v_, beta_, M_, z_):
            out, M_S, z_S = ref.forward(q_, k_, v_, beta_, N, mode=mode, M0=M_, z0=z_)
            return float(np.sum(W_out * out) + np.sum(W_M * M_S) + np.sum(w_z * z_S))

        grads = infini_bwd.backward(q, k, v, beta, N, W_out, W_M, w_z, mode=mode, M0=M0, z0=z0)
        args = [q, k, v, beta, M0, z0]
        for ai, (name, g) in enumerate(zip(("q", "k", "v", "beta", "M0", "z0"), grads)):
            num = np.zeros_like(args[ai])
            eps = 1e-6
            for idx in np.ndindex(args[ai].shape):
                plus = [a.copy() for a in args]
                minus = [a.copy() for a in args]
                plus[ai][idx] += eps
                minus[ai][idx] -= eps
                num[idx] = (loss(*plus) - loss(*minus)) / (2 * eps)
            tol = 1e-6 * max(1.0, float(np.max(np.abs(num))))
            fails += _close(g, num, tol, f"d loss / d {name} (mode {mode})")
    return fails


ALL_PINS.append(pin_backward_finite_differences)
