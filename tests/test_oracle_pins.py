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
