"""Pins of the oracle's token-level pass (``token_level_pass``): checks that
tie it to something other than itself.

Token-level access is the alternative to frame-level access that the pages'
ablation reports as worse (ARL2 summary, §4; §2.2 for the chosen rule): token
t reads the state left by the earlier tokens of the same pass, and the update
of §2.1 runs one token at a time with a per-token decay a_t.  The pins:

* brute force: ``oracle.brute.token_scan`` (scalar loops);
* independent algorithms: the chunked (WY / UT) form below, which solves a
  unit-lower-triangular system per chunk instead of stepping token by token,
  for chunk sizes from 1 to the whole frame with a ragged tail, and its
  rearrangement into one state-free affine map per chunk (the decomposition
  a chunk-parallel kernel computes);
* reductions: one token is the frame-level commit; the first token of any
  frame reads S_{N-1} like every token of a frame-level pass;
* closed forms: beta = 0 gives pure per-token decay; unit keys with
  a = beta = c = 1 store their values exactly, row by row, in order.

Each ``pin_*`` takes an oracle object ``o`` (the module or a broken copy) and
raises AssertionError when ``o`` disagrees.
"""
from __future__ import annotations

import math

import numpy as np

from oracle import brute


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _phi(rng, H, d):
    return tuple(np.eye(d)[None] + _rand(rng, H, d, d) / math.sqrt(d) for _ in range(3))


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:.1e} x {scale:.3g}"


def _case(seed, B=2, L=7, H=2, d=4):
    rng = np.random.default_rng(seed)
    Q, K, V = (_rand(rng, B, L, H, d) for _ in range(3))
    phi = _phi(rng, H, d)
    S = 0.3 * _rand(rng, B, H, d, d)
    a = rng.uniform(0.6, 1.0, (B, H, L))
    beta = rng.uniform(0.0, 1.0, (B, H, L))
    return Q, K, V, phi, S, a, beta


def _mapped(Q, K, V, phi):
    """q'_t, k'_t (unit length), v'_t per (stream, head) as [B, H, L, d]."""
    Qh, Kh, Vh = (np.asarray(x, dtype=np.float64).transpose(0, 2, 1, 3) for x in (Q, K, V))
    Qp = np.einsum("bhli,hij->bhlj", Qh, phi[0])
    Kt = np.einsum("bhli,hij->bhlj", Kh, phi[1])
    Vp = np.einsum("bhli,hij->bhlj", Vh, phi[2])
    return Qp, Kt / np.linalg.norm(Kt, axis=-1, keepdims=True), Vp


def chunked_scan(S0, Qp, Kp, Vp, a, beta, c, chunk):
    """Inter part of a token-level pass for one (stream, head), chunk by chunk.

    Within a chunk with entry state S_0 and g_t = a_1 ... a_t (g_0 = 1), the
    step S_t = a_t S_{t-1} + k_t^T u_t with u_t = c beta_t (v_t - k_t S_{t-1})
    unrolls to S_{t-1} = g_{t-1} S_0 + sum_{s<t} (g_{t-1} / g_s) k_s^T u_s, so
    the rows u_t solve the unit-lower-triangular system

        u_t + c beta_t sum_{s<t} (g_{t-1}/g_s)(k_t . k_s) u_s
            = c beta_t (v_t - g_{t-1} k_t S_0),

    the outputs are o_t = g_{t-1} q_t S_0 + sum_{s<t} (g_{t-1}/g_s)(q_t . k_s) u_s
    and the exit state is g_C S_0 + sum_s (g_C/g_s) k_s^T u_s.  The ratios
    g_{t-1}/g_s are products of a over s < r < t, never quotients."""
    L = Qp.shape[0]
    S = np.array(S0, dtype=np.float64)
    O = np.empty((L, S.shape[1]))
    for c0 in range(0, L, chunk):
        q, k, v = Qp[c0:c0 + chunk], Kp[c0:c0 + chunk], Vp[c0:c0 + chunk]
        ac, w = a[c0:c0 + chunk], c * beta[c0:c0 + chunk]
        n = q.shape[0]
        # G[t, s] = prod of a over s < r < t (0-based in the chunk: r = s+1 .. t-1)
        G = np.zeros((n, n))
        for t in range(n):
            for s in range(t):
                G[t, s] = np.prod(ac[s + 1:t])
        g_prev = np.array([np.prod(ac[:t]) for t in range(n)])        # g_{t-1}
        g_tail = np.array([np.prod(ac[s + 1:]) for s in range(n)])    # g_C / g_s
        A = np.eye(n) + w[:, None] * (G * (k @ k.T))
        rhs = w[:, None] * (v - g_prev[:, None] * (k @ S))
        U = np.linalg.solve(A, rhs)
        O[c0:c0 + n] = g_prev[:, None] * (q @ S) + (G * (q @ k.T)) @ U
        S = np.prod(ac) * S + (g_tail[:, None] * k).T @ U
    return O, S


def affine_chunk_scan(S0, Qp, Kp, Vp, a, beta, c, chunk):
    """The same pass with the entering state taken out of each chunk's work:
    with W = A^-1 diag(c beta g_prev) K and U' = A^-1 diag(c beta) V (A as in
    ``chunked_scan``), every chunk is the affine map

        S_next = (g_C I - Kt^T W) S + Kt^T U',     Kt = diag(g_C / g_s) K,
        O      = (diag(g_prev) Q - P W) S + P U',  P = G * (Q K^T) (strictly lower),

    whose four operands need no state; only S_next = M S + N runs in
    sequence."""
    L, dk = Qp.shape
    maps = []
    for c0 in range(0, L, chunk):
        q, k, v = Qp[c0:c0 + chunk], Kp[c0:c0 + chunk], Vp[c0:c0 + chunk]
        ac, w = a[c0:c0 + chunk], c * beta[c0:c0 + chunk]
        n = q.shape[0]
        G = np.zeros((n, n))
        for t in range(n):
            for s in range(t):
                G[t, s] = np.prod(ac[s + 1:t])
        g_prev = np.array([np.prod(ac[:t]) for t in range(n)])
        g_tail = np.array([np.prod(ac[s + 1:]) for s in range(n)])
        Ainv = np.linalg.inv(np.eye(n) + w[:, None] * (G * (k @ k.T)))
        W = Ainv @ ((w * g_prev)[:, None] * k)
        Up = Ainv @ (w[:, None] * v)
        Kt = g_tail[:, None] * k
        P = G * (q @ k.T)
        maps.append((np.prod(ac) * np.eye(dk) - Kt.T @ W, Kt.T @ Up, g_prev[:, None] * q - P @ W, P @ Up))
    S = np.array(S0, dtype=np.float64)
    outs = []
    for M, N, Qt, Ot in maps:  # the only sequential part
        outs.append(Qt @ S + Ot)
        S = M @ S + N
    return np.concatenate(outs), S


# ---------------------------------------------------------------- pins
def pin_token_brute(o):
    Q, K, V, phi, S, a, beta = _case(41, B=2, L=5, H=2, d=3)
    for c in (1.0, 0.5):
        O, Sn = o.token_level_pass(S, Q, K, V, phi, a, beta, c)
        Ob, Sb = brute.token_scan(S, Q, K, V, phi, a, beta, c)
        intra = np.asarray(brute.softmax_attention(Q, K, V))
        _close(O, intra + np.asarray(Ob), 1e-12, f"token-level output vs brute force (c={c:g})")
        _close(Sn, Sb, 1e-12, f"token-level state vs brute force (c={c:g})")


def pin_token_chunked_form(o):
    Q, K, V, phi, S, a, beta = _case(42, B=1, L=11, H=2, d=5)
    O, Sn = o.token_level_pass(S, Q, K, V, phi, a, beta, 1.0)
    Oi = O - o.intra_softmax(Q, K, V)
    Qp, Kp, Vp = _mapped(Q, K, V, phi)
    for chunk in (1, 2, 3, 4, 11):  # 3 and 4 leave a ragged last chunk
        for h in range(2):
            Oc, Sc = chunked_scan(S[0, h], Qp[0, h], Kp[0, h], Vp[0, h], a[0, h], beta[0, h], 1.0, chunk)
            _close(Oi[0, :, h], Oc, 1e-11, f"output vs chunked form (chunk {chunk})")
            _close(Sn[0, h], Sc, 1e-11, f"state vs chunked form (chunk {chunk})")


def pin_token_affine_chunk_maps(o):
    Q, K, V, phi, S, a, beta = _case(48, B=1, L=10, H=1, d=6)
    O, Sn = o.token_level_pass(S, Q, K, V, phi, a, beta, 0.8)
    Oi = O - o.intra_softmax(Q, K, V)
    Qp, Kp, Vp = _mapped(Q, K, V, phi)
    for chunk in (3, 4, 10):
        Oc, Sc = affine_chunk_scan(S[0, 0], Qp[0, 0], Kp[0, 0], Vp[0, 0], a[0, 0], beta[0, 0], 0.8, chunk)
        _close(Oi[0, :, 0], Oc, 1e-11, f"output vs chunk affine maps (chunk {chunk})")
        _close(Sn[0, 0], Sc, 1e-11, f"state vs chunk affine maps (chunk {chunk})")


def pin_token_single_token_is_frame_level(o):
    Q, K, V, phi, S, a, beta = _case(43, B=2, L=1, H=3, d=4)
    for c in (1.0, 0.25):
        O, Sn = o.token_level_pass(S, Q, K, V, phi, a, beta, c)
        Of, Sf = o.frame_commit(S, Q, K, V, phi, a[:, :, 0], beta, c)
        _close(O, Of, 1e-13, "one token: token-level output = frame-level output")
        _close(Sn, Sf, 1e-13, "one token: token-level state = frame-level state")


def pin_token_first_token_reads_prior_state(o):
    Q, K, V, phi, S, a, beta = _case(44, B=1, L=6, H=2, d=4)
    O, _ = o.token_level_pass(S, Q, K, V, phi, a, beta, 1.0)
    Of = o.frame_query(S, Q, K, V, phi)
    _close(O[:, 0], Of[:, 0], 1e-13, "the first token reads S_{N-1}")
    assert np.max(np.abs(O[:, 1:] - Of[:, 1:])) > 1e-3, "later tokens read the updated state"


def pin_token_beta_zero_is_decay(o):
    Q, K, V, phi, S, a, _ = _case(45, B=1, L=5, H=2, d=4)
    L = Q.shape[1]
    O, Sn = o.token_level_pass(S, Q, K, V, phi, a, np.zeros_like(a), 1.0)
    Qp, _, _ = _mapped(Q, K, V, phi)
    Oi = O - o.intra_softmax(Q, K, V)
    for h in range(2):
        for t in range(L):
            g = np.prod(a[0, h, :t])  # decays of the tokens before t
            _close(Oi[0, t, h], g * (Qp[0, h, t] @ S[0, h]), 1e-13, "beta = 0: o_t = (a_1..a_{t-1}) q'_t S")
        _close(Sn[0, h], np.prod(a[0, h]) * S[0, h], 1e-13, "beta = 0: S_L = (a_1..a_L) S")


def pin_token_unit_keys_store_in_order(o):
    """a = beta = c = 1 and k'_t = e_{i_t}: the step replaces row i_t of the
    state by v'_t, and token t reads the rows written before it."""
    rng = np.random.default_rng(46)
    B, H, d = 1, 1, 6
    rows = [2, 5, 2, 0]  # row 2 is written twice: the later value wins
    L = len(rows)
    K = np.zeros((B, L, H, d))
    for t, i in enumerate(rows):
        K[0, t, 0, i] = 0.5 + t
    Q, V = _rand(rng, B, L, H, d), _rand(rng, B, L, H, d)
    eye = np.eye(d)[None]
    S = _rand(rng, B, H, d, d)
    O, Sn = o.token_level_pass(S, Q, K, V, (eye, eye, eye), np.ones((B, H, L)), np.ones((B, H, L)), 1.0)
    Oi = O - o.intra_softmax(Q, K, V)
    expect = S[0, 0].copy()
    for t, i in enumerate(rows):
        _close(Oi[0, t, 0], Q[0, t, 0] @ expect, 1e-13, f"token {t} reads the rows written before it")
        expect[i] = V[0, t, 0]
    _close(Sn[0, 0], expect, 1e-13, "unit keys store their values in order")


def pin_token_order_matters(o):
    Q, K, V, phi, S, a, beta = _case(47, B=1, L=5, H=1, d=4)
    _, Sn = o.token_level_pass(S, Q, K, V, phi, a, beta, 1.0)
    r = slice(None, None, -1)
    _, Sr = o.token_level_pass(S, Q[:, r], K[:, r], V[:, r], phi, a[:, :, r], beta[:, :, r], 1.0)
    assert np.max(np.abs(Sn - Sr)) > 1e-3, "token-level updates depend on the token order"


TOKEN_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
