"""Token-by-token brute-force evaluation of the Infini-attention forward.

TEST INFRASTRUCTURE ONLY (see ``oracle/infini_ref.py`` for who may use it).

An independent second reading of the same equations, written with scalar
Python loops and ``math.exp`` instead of matrix products, for tiny inputs
only.  Where ``infini_ref`` keeps the memory as the matrix M and vector z,
this file evaluates the linear rule from the closed forms printed on the
explainer page "Leave No Context Behind: Efficient Infinite Context
Transformers with Infini-attention" (section 3, "Compressive Memory"):
M_{s-1} = sum over earlier segments of sigma(K)^T V and
z_{s-1} = sum over earlier tokens of sigma(K), so the memory read of Eq. 7
becomes normalised linear attention over every earlier-segment token.
The delta rule (Eq. 9) has no such closed form; it is evaluated here with
explicit element loops over a list-of-lists memory.
"""

from __future__ import annotations

import math


def sigma(x: float) -> float:
    """ELU(x) + 1 with alpha = 1."""
    return x + 1.0 if x > 0.0 else math.exp(x)


def _sig(beta: float) -> float:
    return 1.0 / (1.0 + math.exp(-beta)) if beta >= 0 else math.exp(beta) / (1.0 + math.exp(beta))


def _dot(a, b):
    acc = 0.0
    for x, y in zip(a, b):
        acc += x * y
    return acc


def local_attention_row(q_t, keys, values, scale):
    """softmax over keys u <= t of the same segment (Eq. 6), one query row, scalar loops."""
    scores = [scale * _dot(q_t, k_u) for k_u in keys]
    m = max(scores)
    w = [math.exp(s - m) for s in scores]
    tot = sum(w)
    dv = len(values[0])
    return [sum(w[u] * values[u][c] for u in range(len(keys))) / tot for c in range(dv)]


def forward_linear_closed_form(q, k, v, beta, N, scale=None):
    """Linear rule via the closed forms: A_mem of token t = normalised linear attention
    over all tokens of earlier segments.  q, k, v: nested lists [B][H][L][d]."""
    B, H, L = len(q), len(q[0]), len(q[0][0])
    dk, dv = len(q[0][0][0]), len(v[0][0][0])
    scale = 1.0 / math.sqrt(dk) if scale is None else scale
    out = [[[None] * L for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            g = _sig(beta[h])
            for t in range(L):
                seg_start = (t // N) * N
                a_dot = local_attention_row(q[b][h][t], k[b][h][seg_start:t + 1], v[b][h][seg_start:t + 1], scale)
                sq = [sigma(x) for x in q[b][h][t]]
                num = [0.0] * dv
                den = 0.0
                for u in range(seg_start):
                    w = _dot(sq, [sigma(x) for x in k[b][h][u]])
                    den += w
                    for c in range(dv):
                        num[c] += w * v[b][h][u][c]
                a_mem = [x / den for x in num] if den != 0.0 else [0.0] * dv
                out[b][h][t] = [g * a_mem[c] + (1.0 - g) * a_dot[c] for c in range(dv)]
    M = [[[[sum(sigma(k[b][h][u][i]) * v[b][h][u][j] for u in range(L)) for j in range(dv)]
           for i in range(dk)] for h in range(H)] for b in range(B)]
    z = [[[sum(sigma(k[b][h][u][i]) for u in range(L)) for i in range(dk)] for h in range(H)] for b in range(B)]
    return out, M, z


def forward_delta_loops(q, k, v, beta, N, scale=None):
    """Delta rule with explicit element loops over a list-of-lists memory (Eq. 7, 9, 10)."""
    B, H, L = len(q), len(q[0]), len(q[0][0])
    dk, dv = len(q[0][0][0]), len(v[0][0][0])
    scale = 1.0 / math.sqrt(dk) if scale is None else scale
    out = [[[None] * L for _ in range(H)] for _ in range(B)]
    Ms, zs = [], []
    for b in range(B):
        Mb, zb = [], []
        for h in range(H):
            g = _sig(beta[h])
            M = [[0.0] * dv for _ in range(dk)]
            z = [0.0] * dk
            for s0 in range(0, L, N):
                s1 = min(s0 + N, L)
                # read with M_{s-1}, z_{s-1}
                for t in range(s0, s1):
                    a_dot = local_attention_row(q[b][h][t], k[b][h][s0:t + 1], v[b][h][s0:t + 1], scale)
                    sq = [sigma(x) for x in q[b][h][t]]
                    den = _dot(sq, z)
                    a_mem = [0.0] * dv
                    if den != 0.0:
                        for c in range(dv):
                            a_mem[c] = sum(sq[i] * M[i][c] for i in range(dk)) / den
                    out[b][h][t] = [g * a_mem[c] + (1.0 - g) * a_dot[c] for c in range(dv)]
                # residual of every token against M_{s-1}, z_{s-1}
                resid = []
                for t in range(s0, s1):
                    sk = [sigma(x) for x in k[b][h][t]]
                    den = _dot(sk, z)
                    r = [0.0] * dv
                    if den != 0.0:
                        for c in range(dv):
                            r[c] = sum(sk[i] * M[i][c] for i in range(dk)) / den
                    resid.append((sk, [v[b][h][t][c] - r[c] for c in range(dv)]))
                for sk, u in resid:
                    for i in range(dk):
                        z[i] += sk[i]
                        for c in range(dv):
                            M[i][c] += sk[i] * u[c]
            Mb.append(M)
            zb.append(z)
        Ms.append(Mb)
        zs.append(zb)
    return out, Ms, zs
