"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that a pin catches each.

This is what makes the pins meaningful: a dropped term, a wrong sign or
index, a transposed operand or a read-after-update must each fail at least
one of them.
"""

import importlib.util
import math

import numpy as np
import pytest

from tests import oracle_pins


def fresh_oracle():
    spec = importlib.util.spec_from_file_location("oracle_mutant", oracle_pins.__file__.replace(
        "tests/oracle_pins.py", "oracle/infini_ref.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def m_elu_without_plus_one(ref):
    ref.elu_plus_one = lambda x: np.where(np.asarray(x) > 0, x, np.exp(np.minimum(x, 0)) - 1.0)


def m_sigma_branch_swapped(ref):
    ref.elu_plus_one = lambda x: np.where(np.asarray(x) >= 0, np.exp(np.minimum(x, 50)), x + 1.0)


def m_exclusive_mask(ref):
    ref.causal_mask = lambda n: np.tril(np.ones((n, n), dtype=bool), k=-1) | (np.arange(n)[:, None] == 0) & (
        np.arange(n)[None, :] == 0)


def m_mask_transposed(ref):
    ref.causal_mask = lambda n: np.triu(np.ones((n, n), dtype=bool))


def m_no_scale(ref):
    orig = ref.causal_softmax_attention
    ref.causal_softmax_attention = lambda Q, K, V, scale: orig(Q, K, V, 1.0)


def m_scale_sqrt_dv(ref):
    orig = ref.causal_softmax_attention
    ref.causal_softmax_attention = lambda Q, K, V, scale: orig(Q, K, V, 1.0 / math.sqrt(V.shape[1] + 1))


def m_gate_swapped(ref):
    orig = ref.gate_weight
    ref.gate_weight = lambda b: 1.0 - orig(b)


def m_linear_update_transposed(ref):
    ref.linear_update = lambda M, z, sk, V: (M + (sk.T @ V).T, z + sk.sum(axis=0))


def m_z_not_updated(ref):
    orig = ref.linear_update
    ref.linear_update = lambda M, z, sk, V: (orig(M, z, sk, V)[0], z)


def m_delta_sign(ref):
    def bad(M, z, sk, V):
        r = ref.memory_retrieval(sk, M, z)
        return M + sk.T @ (V + r), z + sk.sum(axis=0)
    ref.delta_update = bad


def m_delta_uses_new_z(ref):
    def bad(M, z, sk, V):
        z_new = z + sk.sum(axis=0)
        r = ref.memory_retrieval(sk, M, z_new)
        return M + sk.T @ (V - r), z_new
    ref.delta_update = bad


def m_delta_drops_denominator(ref):
    def bad(M, z, sk, V):
        r = sk @ M if np.any(z) else np.zeros((sk.shape[0], M.shape[1]))
        return M + sk.T @ (V - r), z + sk.sum(axis=0)
    ref.delta_update = bad


def m_read_after_update(ref):
    orig = ref.infini_attention_segment

    def bad(Qs, Ks, Vs, M, z, beta_h, mode=0, scale=None):
        _, M2, z2, _ = orig(Qs, Ks, Vs, M, z, beta_h, mode, scale)
        A, _, _, parts = orig(Qs, Ks, Vs, M2, z2, beta_h, mode, scale)
        return A, M2, z2, parts
    ref.infini_attention_segment = bad


def m_retrieval_uses_raw_q(ref):
    def bad(sig_x, M, z):
        x = np.log(np.maximum(sig_x, 1e-300))  # undo sigma on the negative branch only
        num, den = x @ M, sig_x @ z
        out = np.zeros_like(num)
        nz = den != 0
        out[nz] = num[nz] / den[nz, None]
        return out
    ref.memory_retrieval = bad


def m_retrieval_den_squared(ref):
    def bad(sig_x, M, z):
        num, den = sig_x @ M, (sig_x @ z) ** 2
        out = np.zeros_like(num)
        nz = den != 0
        out[nz] = num[nz] / den[nz, None]
        return out
    ref.memory_retrieval = bad


def m_no_max_shift_but_wrong_norm(ref):
    def bad(Q, K, V, scale):
        s = scale * (Q @ K.T)
        s = np.where(ref.causal_mask(Q.shape[0]), s, -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        return (p / Q.shape[0]) @ V
    ref.causal_softmax_attention = bad


def m_segments_off_by_one(ref):
    ref.segment_bounds = lambda L, N: [(s0, min(s0 + N + 1, L)) for s0 in range(0, L, N + 1)]


def m_state_numbers_no_z(ref):
    ref.state_numbers = lambda H, dk, dv: H * dk * dv


def m_flops_full_square(ref):
    def bad(B, H, L, N, dk, dv, mode):
        per = (4 if mode == 0 else 6) * dk * dv
        return B * H * sum((s1 - s0) ** 2 * (dk + dv) + per * (s1 - s0) for s0, s1 in ref.segment_bounds(L, N))
    ref.forward_flops = bad


def _bad_layer(ref, swap_kv=False, head_major_cols=True):
    good_forward = ref.forward

    def layer(x, w_qkv, w_o, beta, H, N, mode=0, M0=None, z0=None, dk=128, round_intermediates=True, scale=None):
        x, w_qkv, w_o = (np.asarray(t, dtype=np.float64) for t in (x, w_qkv, w_o))
        B, L, D = x.shape
        qkv = x @ w_qkv

        def heads(block):
            cols = qkv[:, :, block * H * dk:(block + 1) * H * dk]
            if head_major_cols:
                return cols.reshape(B, L, H, dk).transpose(0, 2, 1, 3)
            return cols.reshape(B, L, dk, H).transpose(0, 3, 1, 2)

        kb, vb = (2, 1) if swap_kv else (1, 2)
        out, M, z = good_forward(heads(0), heads(kb), heads(vb), beta, N, mode=mode, M0=M0, z0=z0, scale=scale)
        return out.transpose(0, 2, 1, 3).reshape(B, L, H * dk) @ w_o, M, z

    return layer


def m_layer_k_v_swapped(ref):
    ref.layer_forward = _bad_layer(ref, swap_kv=True)


def m_layer_head_columns_interleaved(ref):
    ref.layer_forward = _bad_layer(ref, head_major_cols=False)


def m_bf16_truncates(ref):
    def bad(a):
        u = np.asarray(a, dtype=np.float32).view(np.uint32)
        return (u & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)
    ref.bf16_round = bad


def m_decode_folds_every_token(ref):
    good = ref.decode_step

    def bad(q_t, k_t, v_t, k_cache, v_cache, beta, M, z, pos, mode=0, fold=False, scale=None):
        return good(q_t, k_t, v_t, k_cache, v_cache, beta, M, z, pos, mode=mode, fold=True, scale=scale)
    ref.decode_step = bad


def m_rope_half_split_pairs(ref):
    def bad(x, positions, base=10000.0):
        x = np.asarray(x, dtype=np.float64)
        d = x.shape[1]
        h = d // 2
        ang = np.asarray(positions, dtype=np.float64)[:, None] * base ** (-2.0 * np.arange(h) / d)[None, :]
        c, s = np.cos(ang), np.sin(ang)
        out = np.empty_like(x)
        out[:, :h] = x[:, :h] * c - x[:, h:] * s
        out[:, h:] = x[:, :h] * s + x[:, h:] * c
        return out
    ref.rope = bad


def m_rope_applied_to_memory(ref):
    good_segment = ref.infini_attention_segment

    def bad(Qs, Ks, Vs, M, z, beta_h, mode=0, scale=None, q_local=None, k_local=None):
        if q_local is not None:
            Qs, Ks = q_local, k_local
        return good_segment(Qs, Ks, Vs, M, z, beta_h, mode, scale, q_local, k_local)
    ref.infini_attention_segment = bad


MUTANTS = [v for k, v in sorted(globals().items()) if k.startswith("m_")]


@pytest.mark.parametrize("mutate", MUTANTS, ids=lambda f: f.__name__)
def test_pins_catch_mutant(mutate):
    ref = fresh_oracle()
    assert not oracle_pins.run_all(ref), "fresh copy of the oracle must pass"
    mutate(ref)
    bad = oracle_pins.run_all(ref)
    assert bad, f"no pin caught mutation {mutate.__name__}"


@pytest.mark.parametrize("which", ["sigma_prime_one", "no_gate_grad", "every_second_retrieval_grad_dropped"])
def test_backward_pin_catches_mutant(which, monkeypatch):
    """Plausible mistakes in the back-propagation oracle fail the finite-difference pin."""
    from oracle import infini_bwd

    if which == "sigma_prime_one":
        monkeypatch.setattr(infini_bwd, "_sigma_prime", lambda x: np.ones_like(x))
    elif which == "no_gate_grad":
        good = infini_bwd.segment_backward

        def bad(*a, **kw):
            r = good(*a, **kw)
            return r[0], r[1], r[2], 0.0, r[4], r[5]
        monkeypatch.setattr(infini_bwd, "segment_backward", bad)
    else:
        good_rb = infini_bwd._retrieval_backward
        calls = {"n": 0}

        def bad_rb(sig_x, M, z, out, d_out):
            calls["n"] += 1
            d_sig, dM, dz = good_rb(sig_x, M, z, out, d_out)
            # every second retrieval (the delta update's, or every other segment's read) loses its contribution
            return (d_sig * 0.0, dM * 0.0, dz * 0.0) if calls["n"] % 2 == 0 else (d_sig, dM, dz)
        monkeypatch.setattr(infini_bwd, "_retrieval_backward", bad_rb)
    ref = fresh_oracle()
    assert oracle_pins.pin_backward_finite_differences(ref), f"finite-difference pin missed {which}"
