"""The CPU oracle against its pins (brute force, closed forms, invariants)."""
import numpy as np
import pytest

from oracle import arl2_oracle as o
from tests.oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(o)


def _spectral_radius_of_update(L, d, c, alpha, seed):
    """Largest |eigenvalue| of the linear part S -> alpha S - c K'^T diag(beta) K' S."""
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((L, d))
    Kp = K / np.linalg.norm(K, axis=1, keepdims=True)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    G = Kp.T @ (beta[:, None] * Kp)
    lam = np.linalg.eigvalsh(G)
    return float(np.max(np.abs(alpha - c * lam)))


def test_literal_correction_expands_when_tokens_exceed_width():
    """Reading of the correction coefficient: with c = 1 and L >> d the frame map
    has spectral radius well above 1 (the state grows every frame); with c = 1/L
    it is a contraction for alpha in (0, 1) and beta in [0, 1]."""
    L, d = 1560, 128
    assert _spectral_radius_of_update(L, d, 1.0, 0.88, 1) > 5.0
    for seed in range(3):
        assert _spectral_radius_of_update(L, d, 1.0 / L, 0.88, seed) < 1.0
    # and on the tiny stream shape (L = 16 < d = 32) the literal form is stable
    assert _spectral_radius_of_update(16, 32, 1.0, 0.88, 2) <= 1.0


def test_stream_state_growth_matches_reading():
    rng = np.random.default_rng(3)
    B, L, H, d, F = 1, 96, 1, 8, 6
    eye = np.eye(d)[None]
    phi = (eye, eye, eye)
    frames = [tuple(rng.standard_normal((B, L, H, d)) for _ in range(3)) for _ in range(F)]
    gates = lambda n: (np.full((B, H), 0.88), np.full((B, H, L), 0.5))
    qkv = lambda n, p: frames[n]
    _, lit = o.stream_reference((qkv, gates), F, 0, 1.0, phi, keep_outputs=False)
    _, mean = o.stream_reference((qkv, gates), F, 0, 1.0 / L, phi, keep_outputs=False)
    n_lit = [np.linalg.norm(S) for S in lit]
    n_mean = [np.linalg.norm(S) for S in mean]
    assert n_lit[-1] > 1e3 * n_lit[0]
    assert max(n_mean) < 10.0


def test_stream_reference_chains_the_states_it_reads():
    """A closed form of the stream loop.  With identity maps, c = 1, beta = 1
    and a commit whose L = d keys are the unit vectors (K' = I), the correction
    replaces the state: S_n = alpha S_{n-1} + (V_n - S_{n-1}).  The query passes
    use the same Q, K, V in every frame, so the intra-frame part of their output
    is the same each frame and O(frame n) - O(frame 0) = Q S_{n-1} (S_0 = 0):
    each frame's queries read the state the previous commit wrote, and the
    commit's own output reads the state before its update."""
    rng = np.random.default_rng(11)
    B, H, d, F, alpha = 1, 1, 8, 5, 0.75
    L = d
    eye = np.eye(d)[None]
    phi = (eye, eye, eye)
    Kc = np.eye(d)[None, :, None, :]  # the commit's keys: token t is e_t
    Vc = [rng.standard_normal((B, L, H, d)) for _ in range(F)]
    Qc = rng.standard_normal((B, L, H, d))
    Qq, Kq, Vq = (rng.standard_normal((B, L, H, d)) for _ in range(3))

    def qkv(n, p):
        return (Qq, Kq, Vq) if p == 0 else (Qc, Kc, Vc[n])

    gates = lambda n: (np.full((B, H), alpha), np.ones((B, H, L)))
    outs, states = o.stream_reference((qkv, gates), F, 1, 1.0, phi)
    S = np.zeros((d, d))
    expected = []
    for n in range(F):
        S = alpha * S + (Vc[n][0, :, 0, :] - S)
        expected.append(S.copy())
    for n in range(F):
        np.testing.assert_allclose(states[n][0, 0], expected[n], rtol=0, atol=1e-12)
    for n in range(1, F):
        read_out = outs[n][0] - outs[0][0]  # the query pass of frame n minus that of frame 0
        np.testing.assert_allclose(read_out[0, :, 0, :], Qq[0, :, 0, :] @ expected[n - 1], rtol=0, atol=1e-12)
    # the commit of frame n reads S_{n-1}: its keys are the unit vectors, so its
    # attention weights are softmax(Q_c I / sqrt(d)) = A, the same each frame,
    # and O_commit(n) = A V_n + Q_c S_{n-1}
    e = np.exp(Qc[0, :, 0, :] / np.sqrt(d))
    A = e / e.sum(axis=1, keepdims=True)
    for n in range(F):
        prev = expected[n - 1] if n else np.zeros((d, d))
        np.testing.assert_allclose(outs[n][1][0, :, 0, :], A @ Vc[n][0, :, 0, :] + Qc[0, :, 0, :] @ prev,
                                   rtol=0, atol=1e-12)
