"""fp64 CPU oracle for the gradients of the Infini-attention forward (back-propagation
through time over the recurrent memory).

TEST INFRASTRUCTURE ONLY, like ``infini_ref``: nothing on the product path imports it.

The explainer page "Leave No Context Behind: Efficient Infinite Context Transformers
with Infini-attention" (section 3, "Training infrastructure") states that the models are
trained with back-propagation through time over the compressive memory; the pages give
no backward formulas.  This module is the derivative of ``infini_ref.forward`` written out
by the chain rule, segment by segment in reverse order, with the forward's conventions
(zero retrieval row where the denominator is exactly 0; sigma'(x) = 1 for x > 0 and e^x
otherwise).  It is pinned to central finite differences of the forward, not to itself.

Loss convention: the caller supplies the gradients of a scalar loss with respect to the
outputs ``out`` and to the final state ``M_S``, ``z_S``; ``backward`` returns the
gradients with respect to q, k, v, beta and the initial state M_0, z_0.
"""

from __future__ import annotations

import math

import numpy as np

from oracle import infini_ref as R


def _sigma_prime(x: np.ndarray) -> np.ndarray:
    """Derivative of sigma = ELU + 1 (alpha = 1): 1 above zero, e^x at or below."""
    return np.where(x > 0.0, 1.0, np.exp(np.minimum(x, 0.0)))


def _retrieval_backward(sig_x, M, z, out, d_out):
    """Gradients of out = sigma(X) M / (sigma(X) z) (Eq. 7; zero rows where the denominator
    is 0) with respect to sigma(X), M and z, given d_out."""
    den = sig_x @ z
    nz = den != 0.0
    d_num = np.zeros_like(d_out)
    d_den = np.zeros(den.shape)
    d_num[nz] = d_out[nz] / den[nz, None]
    d_den[nz] = -np.sum(d_out[nz] * out[nz], axis=1) / den[nz]
    d_sig = d_num @ M.T + d_den[:, None] * z[None, :]
    return d_sig, sig_x.T @ d_num, sig_x.T @ d_den


def segment_backward(Qs, Ks, Vs, M, z, beta_h, mode, scale, d_A, d_Mn, d_zn):
    """Reverse of one segment of one head (Eq. 6, 7, 10 and Eq. 8 / Eq. 9).

    Inputs: the segment's Q, K, V, the memory M_{s-1}, z_{s-1} it read, and the gradients
    of the loss with respect to its output A and to M_s, z_s.  Returns the gradients with
    respect to Q, K, V, beta_h, M_{s-1}, z_{s-1}.
    """
    n = Qs.shape[0]
    sig_q, sig_k = R.elu_plus_one(Qs), R.elu_plus_one(Ks)
    g = R.gate_weight(beta_h)
    # forward quantities of this segment
    S = scale * (Qs @ Ks.T)
    S = np.where(R.causal_mask(n), S, -np.inf)
    P = np.exp(S - S.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    a_dot = P @ Vs
    a_mem = R.memory_retrieval(sig_q, M, z)
    # gate (Eq. 10)
    d_beta = float(np.sum(d_A * (a_mem - a_dot))) * g * (1.0 - g)
    d_dot, d_mem = (1.0 - g) * d_A, g * d_A
    # local causal attention (Eq. 6)
    dV = P.T @ d_dot
    dP = d_dot @ Vs.T
    dS = P * (dP - np.sum(dP * P, axis=1, keepdims=True))
    dQ = scale * (dS @ Ks)
    dK = scale * (dS.T @ Qs)
    # memory read (Eq. 7)
    d_sig_q, dM, dz = _retrieval_backward(sig_q, M, z, a_mem, d_mem)
    dQ += d_sig_q * _sigma_prime(Qs)
    # memory update (Eq. 8 / Eq. 9): M_s = M + sigma(K)^T U, z_s = z + sum_t sigma(K_t)
    dM = dM + d_Mn
    dz = dz + d_zn
    d_sig_k = np.ones((n, 1)) * d_zn[None, :]
    if mode == R.LINEAR:
        U = Vs
        d_sig_k += U @ d_Mn.T
        dV += sig_k @ d_Mn
    else:
        Rk = R.memory_retrieval(sig_k, M, z)  # retrieval with M_{s-1}, z_{s-1}
        U = Vs - Rk
        d_sig_k += U @ d_Mn.T
        dU = sig_k @ d_Mn
        dV += dU
        d_sig_r, dM_r, dz_r = _retrieval_backward(sig_k, M, z, Rk, -dU)
        d_sig_k += d_sig_r
        dM += dM_r
        dz += dz_r
    dK += d_sig_k * _sigma_prime(Ks)
    return dQ, dK, dV, d_beta, dM, dz


def backward(q, k, v, beta, N, d_out, d_M_final=None, d_z_final=None, mode=R.LINEAR, M0=None, z0=None, scale=None):
    """Gradients of a scalar loss through the whole-sequence forward (``infini_ref.forward``).

    d_out: [B, H, L, dv] = dLoss/d out; d_M_final [B, H, dk, dv], d_z_final [B, H, dk] =
    dLoss/d M_S, z_S (zero when omitted).  Returns (dq, dk, dv, dbeta, dM0, dz0).
    """
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    beta = np.asarray(beta, dtype=np.float64)
    d_out = np.asarray(d_out, dtype=np.float64)
    B, H, L, dk = q.shape
    dv = v.shape[3]
    scale = 1.0 / math.sqrt(dk) if scale is None else scale
    M_init = np.zeros((B, H, dk, dv)) if M0 is None else np.asarray(M0, dtype=np.float64)
    z_init = np.zeros((B, H, dk)) if z0 is None else np.asarray(z0, dtype=np.float64)
    gq, gk, gv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    gbeta = np.zeros(H)
    gM0, gz0 = np.zeros((B, H, dk, dv)), np.zeros((B, H, dk))
    bounds = R.segment_bounds(L, N)
    for b in range(B):
        for h in range(H):
            # forward once more to keep the state entering every segment
            states = []
            M, z = M_init[b, h].copy(), z_init[b, h].copy()
            for s0, s1 in bounds:
                states.append((M, z))
                _, M, z, _ = R.infini_attention_segment(q[b, h, s0:s1], k[b, h, s0:s1], v[b, h, s0:s1], M, z,
                                                        beta[h], mode, scale)
            dMn = np.zeros((dk, dv)) if d_M_final is None else np.array(d_M_final[b, h], dtype=np.float64)
            dzn = np.zeros(dk) if d_z_final is None else np.array(d_z_final[b, h], dtype=np.float64)
            for si in range(len(bounds) - 1, -1, -1):
                s0, s1 = bounds[si]
                Ms, zs = states[si]
                dQ, dK, dV, db, dMn, dzn = segment_backward(q[b, h, s0:s1], k[b, h, s0:s1], v[b, h, s0:s1], Ms, zs,
                                                           beta[h], mode, scale, d_out[b, h, s0:s1], dMn, dzn)
                gq[b, h, s0:s1], gk[b, h, s0:s1], gv[b, h, s0:s1] = dQ, dK, dV
                gbeta[h] += db
            gM0[b, h], gz0[b, h] = dMn, dzn
    return gq, gk, gv, gbeta, gM0, gz0
