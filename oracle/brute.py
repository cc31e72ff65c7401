"""Brute-force restatement of the ARL2 hybrid layer -- TEST INFRASTRUCTURE ONLY.

Pure-Python loops over scalars (math.exp, explicit sums), for inputs of a
few tokens and channels.  It exists to pin the vectorised oracle in
``arl2_oracle.py``: the two are written independently, and the update is
accumulated here token by token as a sum of rank-1 outer products, each token
reading the same pre-update state (ARL2 summary, §2.2, frame-level access),
rather than as one matrix product.  A transposed operand, a dropped gate or a
state read after the write changes the result of one of the two but not of
the other.

Inputs are nested Python lists or numpy arrays in the C-ABI layouts
(Q [B, L, H, d], phi [H, d, d], S [B, H, d, d], alpha [B, H], beta [B, H, L]).
"""
from __future__ import annotations

import math

__all__ = ["softmax_attention", "frame_commit", "sequential_commit", "token_scan"]


def _dot(a, b):
    return sum(float(x) * float(y) for x, y in zip(a, b))


def _vecmat(x, M):
    """row vector x times matrix M (M[i][j]): sum_i x_i M[i][j]."""
    n_out = len(M[0])
    return [sum(float(x[i]) * float(M[i][j]) for i in range(len(x))) for j in range(n_out)]


def softmax_attention(Q, K, V, scale=None):
    """softmax(q k^T * scale) v for every query token, stream and head."""
    B, Lq, H, d = len(Q), len(Q[0]), len(Q[0][0]), len(Q[0][0][0])
    Lk = len(K[0])
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out = [[[None] * H for _ in range(Lq)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            for i in range(Lq):
                logits = [_dot(Q[b][i][h], K[b][j][h]) * scale for j in range(Lk)]
                top = max(logits)
                w = [math.exp(s - top) for s in logits]
                z = sum(w)
                out[b][i][h] = [sum(w[j] * float(V[b][j][h][c]) for j in range(Lk)) / z
                                for c in range(len(V[0][0][0]))]
    return out


def _mapped_token(K, V, phi_k, phi_v, b, t, h):
    kt = _vecmat(K[b][t][h], phi_k[h])
    norm = math.sqrt(sum(x * x for x in kt))
    kp = [x / max(norm, 1e-12) for x in kt]
    vp = _vecmat(V[b][t][h], phi_v[h])
    return kp, vp


def frame_commit(S, Q, K, V, phi, alpha, beta, corr_scale=1.0, scale=None):
    """Output of the clean pass and the frame-level state write.

    O[t] = softmax part + (q_t phi_q) S_{N-1};
    S_N = alpha S_{N-1} + c * sum_t beta_t k'_t (v'_t - k'_t S_{N-1})^T,
    every token using the same S_{N-1}."""
    phi_q, phi_k, phi_v = phi
    B, L, H, d = len(Q), len(Q[0]), len(Q[0][0]), len(Q[0][0][0])
    intra = softmax_attention(Q, K, V, scale)
    O = [[[None] * H for _ in range(L)] for _ in range(B)]
    S_new = []
    for b in range(B):
        S_b = []
        for h in range(H):
            Sp = [[float(x) for x in row] for row in S[b][h]]
            dv = len(Sp[0])
            for t in range(L):
                qp = _vecmat(Q[b][t][h], phi_q[h])
                inter = _vecmat(qp, Sp)
                O[b][t][h] = [intra[b][t][h][c] + inter[c] for c in range(dv)]
            acc = [[0.0] * dv for _ in range(d)]
            for t in range(L):
                kp, vp = _mapped_token(K, V, phi_k, phi_v, b, t, h)
                pred = _vecmat(kp, Sp)            # k'_t S_{N-1}
                bt = float(beta[b][h][t])
                for i in range(d):
                    for j in range(dv):
                        acc[i][j] += bt * kp[i] * (vp[j] - pred[j])
            a = float(alpha[b][h])
            S_b.append([[a * Sp[i][j] + corr_scale * acc[i][j] for j in range(dv)]
                        for i in range(d)])
        S_new.append(S_b)
    return O, S_new


def sequential_commit(S, K, V, phi, alpha, beta, corr_scale=1.0):
    """Token-level access, the alternative the pages' ablation rejects
    (ARL2 summary, §4, ablations): each token's delta step reads the state
    left by the previous token, and the frame's decay is applied once at the
    start.  Used only to show that the frame-level rule is a different
    function, not as a reference for the GPU path."""
    _, phi_k, phi_v = phi
    B, L, H = len(K), len(K[0]), len(K[0][0])
    S_new = []
    for b in range(B):
        S_b = []
        for h in range(H):
            a = float(alpha[b][h])
            Sp = [[a * float(x) for x in row] for row in S[b][h]]
            d, dv = len(Sp), len(Sp[0])
            for t in range(L):
                kp, vp = _mapped_token(K, V, phi_k, phi_v, b, t, h)
                pred = _vecmat(kp, Sp)
                bt = float(beta[b][h][t])
                for i in range(d):
                    for j in range(dv):
                        Sp[i][j] += corr_scale * bt * kp[i] * (vp[j] - pred[j])
            S_b.append(Sp)
        S_new.append(S_b)
    return S_new


def token_scan(S, Q, K, V, phi, alpha_tok, beta, corr_scale=1.0):
    """Inter-frame part of a token-level pass, in scalar loops: token t reads
    the state that tokens 1..t-1 of the same pass left, then writes its own
    delta step (ARL2 summary, §2.1 state update applied one token at a time,
    the access rule of the §4 ablation):

        o_t[j]   = sum_i q'_t[i] S[i][j];
        S[i][j] <- a_t S[i][j] + c beta_t k'_t[i] (v'_t[j] - sum_m k'_t[m] S[m][j]),

    the prediction taken before the update of the step.  Returns (O_inter as
    [B][L][H][d_v] lists, the final state as [B][H][d][d_v] lists)."""
    phi_q, phi_k, phi_v = phi
    B, L, H = len(K), len(K[0]), len(K[0][0])
    O = [[[None] * H for _ in range(L)] for _ in range(B)]
    S_out = []
    for b in range(B):
        S_b = []
        for h in range(H):
            St = [[float(x) for x in row] for row in S[b][h]]
            d, dv = len(St), len(St[0])
            for t in range(L):
                qp = _vecmat(Q[b][t][h], phi_q[h])
                O[b][t][h] = _vecmat(qp, St)
                kp, vp = _mapped_token(K, V, phi_k, phi_v, b, t, h)
                pred = _vecmat(kp, St)
                a, w = float(alpha_tok[b][h][t]), corr_scale * float(beta[b][h][t])
                St = [[a * St[i][j] + w * kp[i] * (vp[j] - pred[j]) for j in range(dv)] for i in range(d)]
            S_b.append(St)
        S_out.append(S_b)
    return O, S_out
