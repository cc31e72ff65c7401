"""Pins of the oracle's attention block (projections around the hybrid layer,
and the commit's gates from the tokens) to facts that do not come from the
block code itself: identity projections reduce it to the layer, distinct
column blocks must land on Q, K and V in that order, the gates' pooling and
layout against scalar loops, zero gate weights, and token permutation."""
import numpy as np
import pytest

from oracle import arl2_oracle as o
from hybrid_linear_attention_arl2_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _case(L=12, H=2, d=16, seed=3):
    cfg = W.Config(92, "block-pin", 1, H, d, L, 2, 1, "f32", corr_scale=1.0)
    wl = W.Workload(cfg, seed=seed)
    return cfg, wl, wl.block_input(0, 0, 0), wl.block_weights(0), wl.phi(0)


def test_identity_projections_reduce_to_the_layer():
    cfg, wl, X, (_, _, w_gate), phi = _case()
    B, L, D = X.shape
    H, d = cfg.heads, cfg.head_dim
    eye = np.eye(D)
    w_qkv = np.concatenate([eye, 2.0 * eye, 3.0 * eye], axis=1)  # Q = X, K = 2X, V = 3X
    rng = np.random.default_rng(0)
    S = rng.standard_normal((B, H, d, d)) * 0.1
    Xr = X.reshape(B, L, H, d).astype(np.float64)
    Y = o.block_query(S, X, (w_qkv, eye, w_gate), phi)
    ref = o.frame_query(S, Xr, 2.0 * Xr, 3.0 * Xr, phi).reshape(B, L, D)
    np.testing.assert_allclose(Y, ref, rtol=0, atol=1e-12)
    alpha, beta = o.block_gates(X, w_gate, H)
    Yc, Sc = o.block_commit(S, X, (w_qkv, eye, w_gate), phi, 0.5)
    refc, Sref = o.frame_commit(S, Xr, 2.0 * Xr, 3.0 * Xr, phi, alpha, beta, 0.5)
    np.testing.assert_allclose(Yc, refc.reshape(B, L, D), rtol=0, atol=1e-12)
    np.testing.assert_allclose(Sc, Sref, rtol=0, atol=1e-12)


def test_output_projection_applies_after_the_layer():
    cfg, wl, X, (w_qkv, w_o, w_gate), phi = _case(seed=5)
    B, L, D = X.shape
    S = np.zeros((B, cfg.heads, cfg.head_dim, cfg.head_dim))
    Q, K, V = o.block_projections(X, w_qkv, cfg.heads)
    O = o.frame_query(S, Q, K, V, phi).reshape(B, L, D)
    # one output element by an explicit sum over the hidden index
    t, j = 3, 7
    want = sum(O[0, t, i] * float(w_o[i, j]) for i in range(D))
    Y = o.block_query(S, X, (w_qkv, w_o, w_gate), phi)
    assert abs(Y[0, t, j] - want) <= 1e-12 * max(1.0, abs(want))


def test_gates_against_scalar_loops():
    cfg, wl, X, (_, _, w_gate), _ = _case(L=9, H=3, d=8, seed=11)
    B, L, D = X.shape
    H = cfg.heads
    alpha, beta = o.block_gates(X, w_gate, H)
    assert alpha.shape == (B, H) and beta.shape == (B, H, L)
    for h in range(H):
        s = 0.0
        for t in range(L):
            s += sum(float(X[0, t, i]) * float(w_gate[i, h]) for i in range(D))
            z = sum(float(X[0, t, i]) * float(w_gate[i, H + h]) for i in range(D))
            assert abs(beta[0, h, t] - 1.0 / (1.0 + np.exp(-z))) <= 1e-12
        assert abs(alpha[0, h] - 1.0 / (1.0 + np.exp(-s / L))) <= 1e-12


def test_zero_gate_weights_give_one_half():
    cfg, wl, X, (_, _, w_gate), _ = _case()
    alpha, beta = o.block_gates(X, np.zeros_like(w_gate), cfg.heads)
    assert np.all(alpha == 0.5) and np.all(beta == 0.5)


def test_token_permutation():
    cfg, wl, X, w, phi = _case(seed=21)
    B, L, D = X.shape
    rng = np.random.default_rng(1)
    S = rng.standard_normal((B, cfg.heads, cfg.head_dim, cfg.head_dim)) * 0.1
    perm = rng.permutation(L)
    Y, S1 = o.block_commit(S, X, w, phi, 1.0 / L)
    Yp, S1p = o.block_commit(S, X[:, perm], w, phi, 1.0 / L)
    np.testing.assert_allclose(Yp, Y[:, perm], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S1p, S1, rtol=1e-10, atol=1e-12)
