"""fp64 CPU oracle for the Infini-attention layer forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
links this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may use it.  It shares no code
with the CUDA library (no kernels, headers, helpers or constants); the two
meet only on seeded inputs produced by ``compressive_memory_transformer_sm_b200.workloads``.

What it computes, step by step, follows the explainer page "Leave No Context
Behind: Efficient Infinite Context Transformers with Infini-attention"
(paper-graph-ui.vercel.app, arXiv 2404.07143), section 3 "Technical
Approach", and uses the paper's equation numbers:

* Eq. 4  recurrent contract  ``O_s, M_s = infini-attention(X_s, M_{s-1})``
* Eq. 6  local causal dot-product attention ``A_dot`` inside one segment
* Eq. 7  memory retrieval ``A_mem = sigma(Q) M_{s-1} / (sigma(Q) z_{s-1})``
         with sigma = ELU + 1
* Eq. 8  linear update  ``M_s = M_{s-1} + sigma(K)^T V``,
         ``z_s = z_{s-1} + sum_t sigma(K_t)``
* Eq. 9  delta update   ``M_s = M_{s-1} + sigma(K)^T (V - sigma(K) M_{s-1} / (sigma(K) z_{s-1}))``
* Eq. 10 gate ``A = sigmoid(beta) * A_mem + (1 - sigmoid(beta)) * A_dot``
* section 3 "Training infrastructure": segment chunking of the length-L
  sequence inside each attention layer (the last segment may be shorter).
* token-level streaming decode (``decode_step``): the abstract's "fast
  streaming inference" read as one new token at a time inside the current
  segment, its keys and values kept in a per-segment cache and folded into
  the memory (Eq. 8 / Eq. 9) once the segment is complete; it must give the
  same outputs and state as the whole-sequence forward.
* Eq. 5  projections ``Q = X W_Q, K = X W_K, V = X W_V`` per head and
  Eq. 11 ``O = [A_1; ...; A_H] W_O`` (section 3, "Multi-Head
  Infini-Attention") for the full layer (``layer_forward``).

Readings taken where the pages are silent or ambiguous (each is also a test):

* softmax scale: Eq. 6 prints ``1/sqrt(d_model)``; the workloads state
  ``1/sqrt(d_key)``, which is the default here (``scale`` overrides it);
* empty memory: ``M_0 = 0, z_0 = 0``; a retrieval whose denominator
  ``sigma(q) z`` is exactly 0 is defined as the zero row (both for A_mem and
  for the delta rule's retrieval term), so at s = 1 the delta update equals
  the linear one;
* ELU uses alpha = 1, so sigma(x) = x + 1 for x > 0 and exp(x) otherwise;
* the delta rule tracks z exactly as the linear rule does, and its retrieval
  uses z_{s-1} (before this segment's keys are added);
* memory is read (A_mem, and the delta retrieval) with M_{s-1}, z_{s-1};
  the update happens after the segment's output;
* the causal mask is inclusive (a query sees itself) and A_dot never looks
  across a segment boundary;
* beta is one scalar per head shared by every batch row, token and channel;
* full layer: the pages fix no precision for the projections; with
  ``round_intermediates`` the layer keeps Q, K, V and the concatenated head
  outputs in bfloat16 between its steps (round to nearest, ties to even), as
  a bf16 implementation stores them; the arithmetic stays fp64.

Everything is evaluated in float64 with NumPy matrix products; there is no
blocking, fusion or reordering beyond what the equations state.
"""

from __future__ import annotations

import math

import numpy as np

LINEAR = 0
DELTA = 1


def elu_plus_one(x: np.ndarray) -> np.ndarray:
    """sigma(x) = ELU(x) + 1 with alpha = 1 (section 3, memory retrieval, Eq. 7)."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0.0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def gate_weight(beta: float) -> float:
    """sigmoid(beta) of the per-head gate (section 3, gating mechanism, Eq. 10)."""
    beta = float(beta)
    if beta >= 0.0:
        return 1.0 / (1.0 + math.exp(-beta))
    e = math.exp(beta)
    return e / (1.0 + e)


def causal_mask(n: int) -> np.ndarray:
    """Allowed (query i, key j) pairs inside one segment: j <= i (Eq. 6, causal masking)."""
    return np.tril(np.ones((n, n), dtype=bool))


def causal_softmax_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """A_dot = softmax(scale * Q K^T) V, row-wise, causal inside the segment (Eq. 6)."""
    scores = scale * (Q @ K.T)
    scores = np.where(causal_mask(Q.shape[0]), scores, -np.inf)
    scores = scores - scores.max(axis=1, keepdims=True)
    p = np.exp(scores)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ V


def memory_retrieval(sig_x: np.ndarray, M: np.ndarray, z: np.ndarray) -> np.ndarray:
    """sigma(X) M / (sigma(X) z), one scalar denominator per row (Eq. 7).

    A row whose denominator is exactly zero (empty memory, z = 0) retrieves
    the zero row -- the reading taken for the first segment.
    """
    num = sig_x @ M
    den = sig_x @ z
    out = np.zeros_like(num)
    nz = den != 0.0
    out[nz] = num[nz] / den[nz, None]
    return out


def linear_update(M: np.ndarray, z: np.ndarray, sig_k: np.ndarray, V: np.ndarray):
    """M_s = M_{s-1} + sigma(K)^T V ; z_s = z_{s-1} + sum_t sigma(K_t) (Eq. 8)."""
    return M + sig_k.T @ V, z + sig_k.sum(axis=0)


def delta_update(M: np.ndarray, z: np.ndarray, sig_k: np.ndarray, V: np.ndarray):
    """M_s = M_{s-1} + sigma(K)^T (V - sigma(K) M_{s-1} / (sigma(K) z_{s-1})) (Eq. 9).

    z is tracked exactly as in the linear rule.
    """
    retrieved = memory_retrieval(sig_k, M, z)
    return M + sig_k.T @ (V - retrieved), z + sig_k.sum(axis=0)


def infini_attention_segment(Qs, Ks, Vs, M, z, beta_h, mode=LINEAR, scale=None, q_local=None, k_local=None):
    """One application of the recurrent layer to one segment of one head (Eq. 4).

    ``q_local`` / ``k_local``: the segment's Q and K with position embeddings,
    used by the local attention only (section 4.1: no position embeddings for
    the compressive memory's keys and queries); Q and K themselves otherwise.
    Returns ``(A, M_s, z_s, parts)`` where ``parts`` holds ``A_dot`` and
    ``A_mem`` for tests that check them separately.
    """
    Qs = np.asarray(Qs, dtype=np.float64)
    Ks = np.asarray(Ks, dtype=np.float64)
    Vs = np.asarray(Vs, dtype=np.float64)
    if scale is None:
        scale = 1.0 / math.sqrt(Qs.shape[1])
    sig_q = elu_plus_one(Qs)
    sig_k = elu_plus_one(Ks)
    a_dot = causal_softmax_attention(Qs if q_local is None else q_local, Ks if k_local is None else k_local, Vs,
                                     scale)
    a_mem = memory_retrieval(sig_q, M, z)
    g = gate_weight(beta_h)
    A = g * a_mem + (1.0 - g) * a_dot
    if mode == LINEAR:
        M_new, z_new = linear_update(M, z, sig_k, Vs)
    elif mode == DELTA:
        M_new, z_new = delta_update(M, z, sig_k, Vs)
    else:
        raise ValueError(f"unknown update mode {mode!r}")
    return A, M_new, z_new, {"A_dot": a_dot, "A_mem": a_mem}


def rope(x, positions, base=10000.0) -> np.ndarray:
    """Rotary position embedding of the rows of x [n, d] (d even) at ``positions`` [n]:
    the pair (x_2i, x_2i+1) is rotated by the angle p * base^(-2i/d).  A reading: the pages
    say only that position embeddings act on the local attention's Q and K (section 4.1);
    rotary embeddings in their original pairwise form are taken as the plainest kind."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[1]
    i = np.arange(d // 2, dtype=np.float64)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * base ** (-2.0 * i / d)[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[:, 0::2], x[:, 1::2]
    out = np.empty_like(x)
    out[:, 0::2] = x0 * c - x1 * s
    out[:, 1::2] = x0 * s + x1 * c
    return out


def segment_bounds(L: int, N: int):
    """Segment chunking: S = ceil(L/N) segments of N tokens, the last one possibly shorter."""
    if L <= 0 or N <= 0:
        raise ValueError("L and N must be positive")
    return [(s0, min(s0 + N, L)) for s0 in range(0, L, N)]


def forward(q, k, v, beta, N, mode=LINEAR, M0=None, z0=None, scale=None, return_parts=False, rope_base=None,
            rope_offset=0):
    """Whole-sequence forward: segment chunking then the recurrence of Eq. 4 per (batch, head).

    q, k: [B, H, L, dk]; v: [B, H, L, dv]; beta: [H]; M0: [B, H, dk, dv]; z0: [B, H, dk].
    ``rope_base``: rotary position embeddings (``rope``) on the local attention's Q and K
    at token positions ``rope_offset + t``; the memory reads and writes un-rotated Q, K.
    Returns ``out [B, H, L, dv]``, ``M_S``, ``z_S`` in float64 (and the A_dot / A_mem
    planes when ``return_parts``).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    B, H, L, dk = q.shape
    dv = v.shape[3]
    M = np.zeros((B, H, dk, dv)) if M0 is None else np.array(M0, dtype=np.float64)
    z = np.zeros((B, H, dk)) if z0 is None else np.array(z0, dtype=np.float64)
    out = np.zeros((B, H, L, dv))
    a_dot_all = np.zeros_like(out) if return_parts else None
    a_mem_all = np.zeros_like(out) if return_parts else None
    for b in range(B):
        for h in range(H):
            Mbh, zbh = M[b, h], z[b, h]
            for s0, s1 in segment_bounds(L, N):
                pe = {}
                if rope_base is not None:
                    pos = rope_offset + np.arange(s0, s1, dtype=np.float64)
                    pe = dict(q_local=rope(q[b, h, s0:s1], pos, rope_base), k_local=rope(k[b, h, s0:s1], pos, rope_base))
                A, Mbh, zbh, parts = infini_attention_segment(
                    q[b, h, s0:s1], k[b, h, s0:s1], v[b, h, s0:s1], Mbh, zbh, beta[h], mode, scale, **pe)
                out[b, h, s0:s1] = A
                if return_parts:
                    a_dot_all[b, h, s0:s1] = parts["A_dot"]
                    a_mem_all[b, h, s0:s1] = parts["A_mem"]
            M[b, h], z[b, h] = Mbh, zbh
    if return_parts:
        return out, M, z, {"A_dot": a_dot_all, "A_mem": a_mem_all}
    return out, M, z


def segment_step(q, k, v, beta, M, z, mode=LINEAR, scale=None):
    """One streaming step: every (batch, head) consumes one segment of n tokens (Eq. 4)."""
    n = np.asarray(q).shape[2]
    return forward(q, k, v, beta, n, mode=mode, M0=M, z0=z, scale=scale)


def state_numbers(H: int, dk: int, dv: int) -> int:
    """Numbers held by the memory of one layer: H (dk dv + dk), independent of L (Table 1)."""
    return H * (dk * dv + dk)


def forward_flops(B: int, H: int, L: int, N: int, dk: int, dv: int, mode: int) -> int:
    """Algorithmic FLOPs of one forward: unmasked causal half of QK^T and PV, memory read and update.

    Per segment of n tokens: n(n+1)(dk+dv) for Eq. 6, 2 n dk dv for the read of
    Eq. 7, 2 n dk dv for sigma(K)^T V and, under the delta rule, 2 n dk dv more
    for sigma(K) M_{s-1}.
    """
    per_mem = (4 if mode == LINEAR else 6) * dk * dv
    total = 0
    for s0, s1 in segment_bounds(L, N):
        n = s1 - s0
        total += n * (n + 1) * (dk + dv) + per_mem * n
    return B * H * total


def memory_trajectory(K, V, N, mode=LINEAR, M0=None, z0=None):
    """States (M_{s-1}, z_{s-1}) entering each segment of one head, and the final (M_S, z_S).

    The update steps of Eq. 8 / Eq. 9 alone, for sampled checks of long inputs
    where the attention of every segment would be too slow on the CPU.
    K: [L, dk], V: [L, dv].
    """
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    dk, dv = K.shape[1], V.shape[1]
    M = np.zeros((dk, dv)) if M0 is None else np.array(M0, dtype=np.float64)
    z = np.zeros(dk) if z0 is None else np.array(z0, dtype=np.float64)
    states = []
    for s0, s1 in segment_bounds(K.shape[0], N):
        states.append((M.copy(), z.copy()))
        sig_k = elu_plus_one(K[s0:s1])
        if mode == LINEAR:
            M, z = linear_update(M, z, sig_k, V[s0:s1])
        else:
            M, z = delta_update(M, z, sig_k, V[s0:s1])
    return states, (M, z)


def segment_output(Qs, Ks, Vs, M, z, beta_h, scale=None):
    """Output A of one segment of one head given the memory (M_{s-1}, z_{s-1}) it reads (Eq. 6, 7, 10)."""
    A, _, _, _ = infini_attention_segment(Qs, Ks, Vs, M, z, beta_h, LINEAR, scale)
    return A


def bf16_round(a) -> np.ndarray:
    """Nearest bfloat16 value (ties to even), as float64: the storage of the
    layer's intermediates in a bf16 implementation (a reading; see the header)."""
    a32 = np.asarray(a, dtype=np.float32)
    u = a32.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


def layer_forward(x, w_qkv, w_o, beta, H, N, mode=LINEAR, M0=None, z0=None, dk=128, round_intermediates=True,
                  scale=None):
    """Multi-head layer around the recurrence: Q, K, V = X W_Q, X W_K, X W_V
    per head (Eq. 5), the whole-sequence ``forward``, then
    O = [A_1; ...; A_H] W_O (Eq. 11).

    x: [B, L, D]; w_qkv: [D, 3 H dk], column blocks Q | K | V, head h in the
    columns h dk .. h dk + dk - 1 of each block; w_o: [H dv, D] with dv = dk,
    row h dv + j multiplying value column j of head h.  Returns
    ``y [B, L, D]``, ``M_S``, ``z_S`` in float64.
    """
    x = np.asarray(x, dtype=np.float64)
    w_qkv = np.asarray(w_qkv, dtype=np.float64)
    w_o = np.asarray(w_o, dtype=np.float64)
    B, L, D = x.shape
    qkv = x @ w_qkv  # Eq. 5 for all heads at once: [B, L, 3 H dk]
    if round_intermediates:
        qkv = bf16_round(qkv)

    def heads(block):
        cols = qkv[:, :, block * H * dk:(block + 1) * H * dk]
        return cols.reshape(B, L, H, dk).transpose(0, 2, 1, 3)  # [B, H, L, dk]

    out, M, z = forward(heads(0), heads(1), heads(2), beta, N, mode=mode, M0=M0, z0=z0, scale=scale)
    a = out.transpose(0, 2, 1, 3).reshape(B, L, H * dk)  # concatenation along the feature axis (Eq. 11)
    if round_intermediates:
        a = bf16_round(a)
    return a @ w_o, M, z


def decode_step(q_t, k_t, v_t, k_cache, v_cache, beta, M, z, pos, mode=LINEAR, fold=False, scale=None):
    """One new token per (batch, head) at position ``pos`` of the current segment.

    q_t, k_t: [B, H, dk]; v_t: [B, H, dv]; k_cache [B, H, N, dk] and v_cache
    [B, H, N, dv] hold the segment's earlier keys and values (updated in
    place: row ``pos`` receives k_t, v_t); M [B, H, dk, dv], z [B, H, dk] are
    the memory entering the segment, M_{s-1} and z_{s-1}.  The token attends
    causally to the segment's keys 0..pos (Eq. 6 for one query row), reads the
    memory (Eq. 7) and blends (Eq. 10).  When the segment is complete
    (pos = N - 1) or ``fold`` is set, the segment's keys and values update the
    memory (Eq. 8 / Eq. 9).  Returns ``out [B, H, dv]``, M, z.
    """
    q_t, k_t, v_t = (np.asarray(t, dtype=np.float64) for t in (q_t, k_t, v_t))
    B, H, dk = q_t.shape
    dv = v_t.shape[2]
    N = k_cache.shape[2]
    scale = 1.0 / math.sqrt(dk) if scale is None else scale
    k_cache[:, :, pos] = k_t
    v_cache[:, :, pos] = v_t
    out = np.zeros((B, H, dv))
    M = np.array(M, dtype=np.float64)
    z = np.array(z, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            keys, vals = k_cache[b, h, :pos + 1], v_cache[b, h, :pos + 1]
            s = scale * (keys @ q_t[b, h])               # scores of the new query row
            p = np.exp(s - s.max())
            a_dot = (p / p.sum()) @ vals
            a_mem = memory_retrieval(elu_plus_one(q_t[b, h][None, :]), M[b, h], z[b, h])[0]
            g = gate_weight(beta[h])
            out[b, h] = g * a_mem + (1.0 - g) * a_dot
    if fold or pos == N - 1:
        for b in range(B):
            for h in range(H):
                sk = elu_plus_one(k_cache[b, h, :pos + 1])
                upd = linear_update if mode == LINEAR else delta_update
                M[b, h], z[b, h] = upd(M[b, h], z[b, h], sk, v_cache[b, h, :pos + 1])
    return out, M, z
