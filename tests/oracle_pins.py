"""Pins of the CPU oracle: checks that tie it to something other than itself.

Each ``pin_*`` function takes an oracle object ``o`` (the module
``oracle.arl2_oracle`` or a deliberately broken copy of it) and raises
AssertionError when ``o`` disagrees with what the pages or the mathematics
fix.  The sources, in the terms the oracle uses:

* brute force: ``oracle.brute`` (scalar loops, token-by-token outer products);
* closed forms: a hand-derived two-token softmax (tests/golden), uniform
  attention when all keys are equal, the single-token frame, orthonormal keys;
* invariants: S = 0 gives O_inter = 0; beta = 0 gives pure decay; a unit key
  with alpha = beta = 1 stores its value exactly; token permutation
  permutes the output and leaves the state; the read-out is linear in Q;
* a library cross-check: torch's scaled_dot_product_attention in float64.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from oracle import brute

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _phi(rng, H, d, ident=1.0):
    return tuple(ident * np.eye(d)[None] + _rand(rng, H, d, d) / math.sqrt(d) for _ in range(3))


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:.1e} x {scale:.3g}"


# ---------------------------------------------------------------- intra branch
def pin_intra_golden(o):
    g = json.load(open(os.path.join(GOLDEN, "intra_two_token.json")))
    O = o.intra_softmax(np.array(g["Q"]), np.array(g["K"]), np.array(g["V"]))
    _close(O, g["O"], g["tolerance"], "two-token closed form")


def pin_intra_brute(o):
    rng = np.random.default_rng(11)
    B, L, H, d = 2, 5, 3, 4
    Q, K, V = (_rand(rng, B, L, H, d) for _ in range(3))
    _close(o.intra_softmax(Q, K, V), brute.softmax_attention(Q, K, V), 1e-12, "intra vs brute force")
    Q2 = 4.0 * _rand(rng, B, 3, H, d)  # a query subset, sharper logits
    _close(o.intra_softmax(Q2, K, V), brute.softmax_attention(Q2, K, V), 1e-12,
           "intra (query subset) vs brute force")


def pin_intra_uniform(o):
    rng = np.random.default_rng(12)
    B, L, H, d = 1, 7, 2, 4
    Q, V = _rand(rng, B, L, H, d), _rand(rng, B, L, H, d)
    K = np.tile(_rand(rng, B, 1, H, d), (1, L, 1, 1))  # all keys equal -> uniform weights
    mean_v = np.broadcast_to(V.mean(axis=1, keepdims=True), V.shape)
    _close(o.intra_softmax(Q, K, V), mean_v, 1e-13, "equal keys give the mean value")


def pin_intra_single_token(o):
    rng = np.random.default_rng(13)
    Q, K, V = (_rand(rng, 1, 1, 2, 8) for _ in range(3))
    _close(o.intra_softmax(Q, K, V), V, 0.0, "one token returns its value")


def pin_intra_sdpa(o):
    import torch
    rng = np.random.default_rng(14)
    B, L, H, d = 1, 9, 2, 8
    Q, K, V = (_rand(rng, B, L, H, d) for _ in range(3))
    t = [torch.from_numpy(x).permute(0, 2, 1, 3) for x in (Q, K, V)]
    ref = torch.nn.functional.scaled_dot_product_attention(*t).permute(0, 2, 1, 3).numpy()
    _close(o.intra_softmax(Q, K, V), ref, 1e-12, "intra vs torch sdpa (float64)")


# ---------------------------------------------------------------- feature maps
def pin_feature_maps(o):
    rng = np.random.default_rng(15)
    B, L, H, d = 1, 6, 2, 5
    Q, K, V = (_rand(rng, B, L, H, d) for _ in range(3))
    eye = np.tile(np.eye(d)[None], (H, 1, 1))
    Qp, Kp, Vp = o.feature_maps(Q, K, V, eye, eye, eye)
    Qh, Kh, Vh = (x.transpose(0, 2, 1, 3) for x in (Q, K, V))
    _close(Qp, Qh, 0.0, "phi_q = I gives Q' = Q")
    _close(Vp, Vh, 0.0, "phi_v = I gives V' = V")
    _close(Kp, Kh / np.linalg.norm(Kh, axis=-1, keepdims=True), 1e-15, "phi_k = I gives K/|K|")
    pq, pk, pv = _phi(rng, H, d)
    Qp, Kp, Vp = o.feature_maps(Q, K, V, pq, pk, pv)
    _close(np.linalg.norm(Kp, axis=-1), np.ones(Kp.shape[:-1]), 1e-14, "K' rows have unit norm")
    # one token and head by hand: q'_j = sum_i q_i phi[i, j]
    qp = [sum(Q[0, 3, 1, i] * pq[1][i, j] for i in range(d)) for j in range(d)]
    _close(Qp[0, 1, 3], qp, 1e-14, "Q' = Q phi_q (row vector times matrix)")


# ---------------------------------------------------------------- read-out
def pin_readout_zero_state(o):
    rng = np.random.default_rng(16)
    B, L, H, d = 2, 5, 2, 4
    Q, K, V = (_rand(rng, B, L, H, d) for _ in range(3))
    phi = _phi(rng, H, d)
    S = np.zeros((B, H, d, d))
    O = o.frame_query(S, Q, K, V, phi)
    _close(O, o.intra_softmax(Q, K, V), 0.0, "S = 0 gives O = O_intra exactly")


def pin_readout_linear(o):
    rng = np.random.default_rng(17)
    B, L, H, d = 1, 4, 2, 3
    Qp = _rand(rng, B, H, L, d)
    S = _rand(rng, B, H, d, d)
    O1 = o.inter_readout(Qp, S)
    _close(o.inter_readout(2.5 * Qp, S), 2.5 * O1, 1e-14, "read-out is linear in Q'")
    # one element by hand: O[b, t, h, j] = sum_i Q'[b, h, t, i] S[b, h, i, j]
    val = sum(Qp[0, 1, 2, i] * S[0, 1, i, 0] for i in range(d))
    _close(O1[0, 2, 1, 0], val, 1e-14, "O_inter = Q' S elementwise")


def pin_query_with_state(o):
    """frame_query against brute force with a non-zero state (alpha = 1, beta = 0 commit
    leaves S as it is, and the brute-force commit computes the same output)."""
    rng = np.random.default_rng(18)
    B, L, H, d = 1, 4, 2, 3
    Q, K, V = (_rand(rng, B, L, H, d) for _ in range(3))
    phi = _phi(rng, H, d)
    S = _rand(rng, B, H, d, d)
    O_b, _ = brute.frame_commit(S, Q, K, V, phi, np.ones((B, H)), np.zeros((B, H, L)))
    _close(o.frame_query(S, Q, K, V, phi), O_b, 1e-12, "query output vs brute force")


# ---------------------------------------------------------------- update
def pin_commit_brute(o):
    rng = np.random.default_rng(19)
    B, L, H, d = 2, 5, 2, 4
    Q, K, V = (_rand(rng, B, L, H, d) for _ in range(3))
    phi = _phi(rng, H, d)
    S = 0.3 * _rand(rng, B, H, d, d)
    alpha = rng.uniform(0.5, 1.0, (B, H))
    beta = rng.uniform(0.0, 1.0, (B, H, L))
    for c in (1.0, 1.0 / L):
        O, Sn = o.frame_commit(S, Q, K, V, phi, alpha, beta, c)
        Ob, Snb = brute.frame_commit(S, Q, K, V, phi, alpha, beta, c)
        _close(O, Ob, 1e-12, f"commit output vs brute force (c={c:g})")
        _close(Sn, Snb, 1e-12, f"commit state vs brute force (c={c:g})")


def pin_commit_beta_zero(o):
    rng = np.random.default_rng(20)
    B, L, H, d = 1, 6, 2, 4
    Q, K, V = (_rand(rng, B, L, H, d) for _ in range(3))
    S = _rand(rng, B, H, d, d)
    alpha = rng.uniform(0.1, 0.9, (B, H))
    _, Sn = o.frame_commit(S, Q, K, V, _phi(rng, H, d), alpha, np.zeros((B, H, L)), 1.0)
    _close(Sn, alpha[..., None, None] * S, 0.0, "beta = 0 gives S_N = alpha S_{N-1}")


def pin_commit_unit_key(o):
    """alpha = beta = 1, one token, c = 1: k' S_N = v' for the stored key."""
    rng = np.random.default_rng(21)
    B, L, H, d = 1, 1, 2, 5
    Q, K, V = (_rand(rng, B, L, H, d) for _ in range(3))
    phi = _phi(rng, H, d)
    S = _rand(rng, B, H, d, d)
    _, Sn = o.frame_commit(S, Q, K, V, phi, np.ones((B, H)), np.ones((B, H, L)), 1.0)
    for h in range(H):
        kt = K[0, 0, h] @ phi[1][h]
        kp = kt / np.linalg.norm(kt)
        vp = V[0, 0, h] @ phi[2][h]
        _close(kp @ Sn[0, h], vp, 1e-12, "unit key recalls its value")


def pin_commit_orthonormal_keys(o):
    """k'_t = e_{i_t} (distinct), beta = 1, c = 1: row i_t of S_N is
    v'_t + (alpha - 1) S_{N-1}[i_t]; other rows decay to alpha S_{N-1}."""
    rng = np.random.default_rng(22)
    B, H, d = 1, 1, 6
    rows = [4, 1, 3]
    L = len(rows)
    K = np.zeros((B, L, H, d))
    for t, i in enumerate(rows):
        K[0, t, 0, i] = 2.0 + t  # any positive length; normalisation makes it e_i
    Q, V = _rand(rng, B, L, H, d), _rand(rng, B, L, H, d)
    eye = np.eye(d)[None]
    phi = (eye, eye, eye)
    S = _rand(rng, B, H, d, d)
    a = 0.7
    _, Sn = o.frame_commit(S, Q, K, V, phi, np.full((B, H), a), np.ones((B, H, L)), 1.0)
    expect = a * S[0, 0].copy()
    for t, i in enumerate(rows):
        expect[i] = V[0, t, 0] + (a - 1.0) * S[0, 0, i]
    _close(Sn[0, 0], expect, 1e-14, "orthonormal-key closed form")


def pin_commit_permutation(o):
    rng = np.random.default_rng(23)
    B, L, H, d = 1, 7, 2, 4
    Q, K, V = (_rand(rng, B, L, H, d) for _ in range(3))
    phi = _phi(rng, H, d)
    S = _rand(rng, B, H, d, d)
    alpha = rng.uniform(0.5, 1.0, (B, H))
    beta = rng.uniform(0.0, 1.0, (B, H, L))
    perm = rng.permutation(L)
    O, Sn = o.frame_commit(S, Q, K, V, phi, alpha, beta, 1.0)
    Op, Snp = o.frame_commit(S, Q[:, perm], K[:, perm], V[:, perm], phi, alpha, beta[:, :, perm], 1.0)
    _close(Op, O[:, perm], 1e-12, "token permutation permutes the output")
    _close(Snp, Sn, 1e-12, "token permutation leaves the state")


def pin_commit_reads_pre_update_state(o):
    """The commit's output equals a query against S_{N-1}, not S_N
    (ARL2 summary, section 2.2, frame-level access)."""
    rng = np.random.default_rng(24)
    B, L, H, d = 1, 5, 2, 4
    Q, K, V = (_rand(rng, B, L, H, d) for _ in range(3))
    phi = _phi(rng, H, d)
    S = _rand(rng, B, H, d, d)
    O, Sn = o.frame_commit(S, Q, K, V, phi, np.full((B, H), 0.9), np.full((B, H, L), 0.5), 1.0)
    _close(O, o.frame_query(S, Q, K, V, phi), 0.0, "commit output reads S_{N-1}")
    assert np.max(np.abs(Sn - S)) > 1e-3


def pin_frame_level_vs_token_level(o):
    """With alpha = 1 and one token, the frame-level rule is the textbook delta
    rule; with several non-orthogonal tokens it differs from sequential
    (token-level) updates."""
    rng = np.random.default_rng(25)
    B, H, d = 1, 1, 4
    phi = _phi(rng, H, d)
    S = _rand(rng, B, H, d, d)
    Q, K, V = (_rand(rng, B, 1, H, d) for _ in range(3))
    _, Sn = o.frame_commit(S, Q, K, V, phi, np.ones((B, H)), np.full((B, H, 1), 0.6), 1.0)
    Ss = brute.sequential_commit(S, K, V, phi, np.ones((B, H)), np.full((B, H, 1), 0.6), 1.0)
    _close(Sn, Ss, 1e-12, "one token: frame-level = delta rule")
    L = 4
    Q, K, V = (_rand(rng, B, L, H, d) for _ in range(3))
    _, Sn = o.frame_commit(S, Q, K, V, phi, np.ones((B, H)), np.full((B, H, L), 0.6), 1.0)
    Ss = np.array(brute.sequential_commit(S, K, V, phi, np.ones((B, H)), np.full((B, H, L), 0.6), 1.0))
    assert np.max(np.abs(Sn - Ss)) > 1e-3, "frame-level access must differ from token-level"


def pin_kv_attention(o):
    rng = np.random.default_rng(26)
    B, L, H, d = 1, 3, 2, 4
    past = [(_rand(rng, B, L, H, d), _rand(rng, B, L, H, d)) for _ in range(2)]
    Q, K, V = (_rand(rng, B, L, H, d) for _ in range(3))
    Kc = np.concatenate([p[0] for p in past] + [K], axis=1)
    Vc = np.concatenate([p[1] for p in past] + [V], axis=1)
    _close(o.kv_attention(Q, Kc, Vc), brute.softmax_attention(Q, Kc, Vc), 1e-12,
           "KV-cache attention vs brute force")
    _close(o.kv_attention(Q, K, V), o.intra_softmax(Q, K, V), 0.0, "empty cache is the intra branch")


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
