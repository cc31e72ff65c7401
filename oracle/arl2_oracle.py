"""CPU oracle for the ARL2 hybrid-attention hot path -- TEST INFRASTRUCTURE ONLY.

Only the tests, the package's ``smoke()`` check and the benchmark's CPU
baseline may import this module.  The CUDA path never calls it, and it shares
no code with the CUDA path: it is the plain definition of what one hybrid
layer computes, in numpy float64, with no blocking, fusion or reordering.

Sources.  "ARL2 summary" below is the technical summary on the page
"Attend Locally, Remember Linearly: Linear Attention as Cross-Frame Memory for
Autoregressive Video Diffusion" (gist.science, German; the Italian, Japanese
and Korean pages of the same site carry the same text).  "ARL2 abstract" is
the authors' English abstract of arXiv 2605.16579v2 as shown on the
fugumt.com paper_check page.

Layouts (those of the C ABI): Q, K, V, O are [B, L, H, d] (token-major);
phi_* are [H, d, d] with Q' = Q @ phi_q; S is [B, H, d_k, d_v]; alpha is
[B, H] (one gate per stream and head for the frame); beta is [B, H, L].

Readings of the pages that this file fixes (each is listed with its reason
in the design notes of the repository):

* the update's lost transposes: the delta term is K'^T diag(beta)(V' - K'S);
* K' is L2-normalised per token, max(||k||, 1e-12) in the denominator; Q'
  and V' are not normalised; the phi maps are plain d x d matrices;
* alpha is one scalar per (stream, head, frame); beta one value per token;
* O = O_intra + O_inter, with no gate or normalisation between them;
* the delta correction carries an explicit coefficient c (``corr_scale``);
  c = 1 is the literal formula, c = 1/L the mean over the frame's tokens.
* token-level access (``token_level_pass``, the rule the ablation rejects):
  the same update one token at a time, with a per-token decay a_t and the
  prediction taken before the token's own decay.

Parity status: the intra branch, the read-out and the update are each pinned
by brute force on tiny inputs, closed forms and invariants (tests marked
"not gpu"); the token-level pass also by an independently derived chunked
form.  The values of a full frame at the benchmark shapes are pinned
only through those same definitions: the pages print no worked numbers.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "feature_maps", "intra_softmax", "inter_readout", "frame_query",
    "frame_commit", "state_update", "kv_attention", "token_level_pass", "stream_reference",
]

EPS_NORM = 1e-12


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _heads_first(x: np.ndarray) -> np.ndarray:
    """[B, L, H, d] -> [B, H, L, d]."""
    return np.ascontiguousarray(x.transpose(0, 2, 1, 3))


def _tokens_first(x: np.ndarray) -> np.ndarray:
    """[B, H, L, d] -> [B, L, H, d]."""
    return np.ascontiguousarray(x.transpose(0, 2, 1, 3))


def feature_maps(Q, K, V, phi_q, phi_k, phi_v):
    """Per-head grouped 1x1 feature maps (ARL2 summary, §2.1, "Anpassung"):
    Q' = Q phi_q, K' = rownorm_2(K phi_k), V' = V phi_v, each [B, H, L, d]."""
    Qh, Kh, Vh = (_heads_first(_f64(t)) for t in (Q, K, V))
    Qp = Qh @ _f64(phi_q)[None]
    Kt = Kh @ _f64(phi_k)[None]
    Vp = Vh @ _f64(phi_v)[None]
    norm = np.sqrt(np.sum(Kt * Kt, axis=-1, keepdims=True))
    Kp = Kt / np.maximum(norm, EPS_NORM)
    return Qp, Kp, Vp


def intra_softmax(Q, K, V, scale=None):
    """Intra-frame branch (ARL2 summary, §2.1, "Intra-Frame-Zweig"): the
    original bidirectional softmax attention over the tokens of one frame,
    on the unmapped Q, K, V; no mask.  Q may hold any subset of the frame's
    query tokens.  Returns [B, Lq, H, d]."""
    Qh, Kh, Vh = (_heads_first(_f64(t)) for t in (Q, K, V))
    d = Qh.shape[-1]
    scale = d ** -0.5 if scale is None else float(scale)
    s = (Qh @ np.swapaxes(Kh, -1, -2)) * scale
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    O = (p @ Vh) / p.sum(axis=-1, keepdims=True)
    return _tokens_first(O)


def inter_readout(Qp, S):
    """Inter-frame read-out (ARL2 summary, §2.1, "Ausgabe"): O_inter = Q' S,
    with Q' [B, H, L, d_k] and S [B, H, d_k, d_v].  Returns [B, L, H, d_v]."""
    return _tokens_first(_f64(Qp) @ _f64(S))


def frame_query(S, Q, K, V, phi, scale=None):
    """One denoising step: O = O_intra + Q' S_{N-1}.  The state is only read
    (ARL2 summary, §2.2, "Clean-Pass-Aktualisierungen"); every token reads the
    same S_{N-1} (§2.2, "Frame-Level-Zugriff")."""
    phi_q, phi_k, phi_v = phi
    Qp = _heads_first(_f64(Q)) @ _f64(phi_q)[None]
    return intra_softmax(Q, K, V, scale) + inter_readout(Qp, S)


def frame_commit(S, Q, K, V, phi, alpha, beta, corr_scale=1.0, scale=None):
    """The clean pass of frame N: the output from S_{N-1}, then the single
    state write of the frame (ARL2 summary, §2.1 "Zustandsaktualisierung" and
    §2.2; ARL2 abstract: update only after the denoised pass, all tokens
    share the pre-update state):

        S_N = alpha_N S_{N-1} + c K'^T diag(beta) (V' - K' S_{N-1}).

    Returns (O [B, L, H, d], S_N [B, H, d, d])."""
    S = _f64(S)
    O = frame_query(S, Q, K, V, phi, scale)
    return O, state_update(S, K, V, phi, alpha, beta, corr_scale)


def state_update(S, K, V, phi, alpha, beta, corr_scale=1.0):
    """The state write of a commit alone (ARL2 summary, §2.1
    "Zustandsaktualisierung"): S_N = alpha S + c K'^T diag(beta)(V' - K' S),
    every token of the frame reading the same S = S_{N-1} (§2.2)."""
    S = _f64(S)
    _, Kp, Vp = feature_maps(K, K, V, *phi)
    R = _f64(beta)[..., None] * (Vp - Kp @ S)
    delta = np.swapaxes(Kp, -1, -2) @ R
    return _f64(alpha)[..., None, None] * S + float(corr_scale) * delta


def kv_attention(Q, K_ctx, V_ctx, scale=None):
    """A softmax layer kept from the teacher, over a growing key-value cache
    (ARL2 summary, §1, KV-cache growth): the queries of frame n attend to the
    clean keys and values of frames 0..n-1 followed by the current pass's own
    keys and values, with no mask.  K_ctx and V_ctx are that concatenation,
    [B, Lk, H, d]."""
    return intra_softmax(Q, K_ctx, V_ctx, scale)


def token_level_pass(S, Q, K, V, phi, alpha_tok, beta, corr_scale=1.0, scale=None):
    """Token-level access: the alternative to frame-level access that the
    pages' ablation reports as worse (ARL2 summary, §4, ablations; §2.2 names
    frame-level access, every token reading S_{N-1}, as the chosen rule).
    Within one pass, token t reads the state left by the tokens before it in
    the same pass, and the update of §2.1 ("Zustandsaktualisierung") is
    applied one token at a time:

        o_t   = O_intra,t + q'_t S^(t-1),          S^(0) = S_{N-1},
        S^(t) = a_t S^(t-1) + c beta_t k'_t^T (v'_t - k'_t S^(t-1)).

    a is a decay per token (``alpha_tok`` [B, H, L]): the frame-level gate
    alpha corresponds to a = (alpha, 1, ..., 1), and a general ``alpha_tok``
    is the per-token gate the pages' wording also allows (§2.1).  The
    prediction k'_t S^(t-1) reads the state before the token's own decay, as
    the frame-level formula reads S_{N-1}.  Returns (O [B, L, H, d],
    S^(L) [B, H, d, d]); a query pass keeps O and drops S^(L), since only the
    clean pass writes the state (§2.2).

    Token by token in order, each step vectorised over streams and heads."""
    St = _f64(S).copy()
    Qp, Kp, Vp = feature_maps(Q, K, V, *phi)
    a, bt, c = _f64(alpha_tok), _f64(beta), float(corr_scale)
    B, H, L, _ = Qp.shape
    Oi = np.empty((B, H, L, St.shape[-1]))
    for t in range(L):
        Oi[:, :, t, :] = np.einsum("bhi,bhij->bhj", Qp[:, :, t, :], St)
        pred = np.einsum("bhi,bhij->bhj", Kp[:, :, t, :], St)
        r = bt[:, :, t, None] * (Vp[:, :, t, :] - pred)
        St = a[:, :, t, None, None] * St + c * Kp[:, :, t, :, None] * r[:, :, None, :]
    return intra_softmax(Q, K, V, scale) + _tokens_first(Oi), St


def stream_reference(inputs, frames, queries, corr_scale, phi, S0=None, scale=None,
                     keep_outputs=True):
    """Run a hybrid layer over a stream: for each frame, ``queries`` query
    passes and one commit.  ``inputs(frame, pas)`` returns (Q, K, V) and
    ``gates(frame)`` the pair (alpha, beta); both are supplied by the caller
    as ``inputs = (qkv_fn, gates_fn)``.  Returns the list of per-frame output
    lists and the list of states S_1..S_F."""
    qkv_fn, gates_fn = inputs
    Q0, _, _ = qkv_fn(0, 0)
    B, L, H, d = Q0.shape
    S = np.zeros((B, H, d, d)) if S0 is None else _f64(S0)
    outs, states = [], []
    for n in range(frames):
        frame_out = []
        for p in range(queries):
            Q, K, V = qkv_fn(n, p)
            O = frame_query(S, Q, K, V, phi, scale)
            frame_out.append(O if keep_outputs else None)
        Q, K, V = qkv_fn(n, queries)
        alpha, beta = gates_fn(n)
        O, S = frame_commit(S, Q, K, V, phi, alpha, beta, corr_scale, scale)
        frame_out.append(O if keep_outputs else None)
        outs.append(frame_out)
        states.append(S)
    return outs, states


# ---------------------------------------------------------------- attention block
def block_projections(X, w_qkv, heads):
    """Q, K, V of a hybrid attention block: the frozen pretrained projections
    in front of both branches (ARL2 summary, §2.1), X [B, L, D] times the
    three column blocks of w_qkv [D, 3D], each reshaped to [B, L, H, D/H]."""
    X, w = _f64(X), _f64(w_qkv)
    B, L, D = X.shape
    d = D // heads
    QKV = X @ w
    return tuple(QKV[..., i * D:(i + 1) * D].reshape(B, L, heads, d) for i in range(3))


def block_gates(X, w_gate, heads):
    """The commit's gates from the tokens (ARL2 summary, §2.1: alpha and beta
    are learned projections of the tokens).  Reading of this build: the first
    H columns of X w_gate give alpha from the frame's mean token, one per head
    (head-wise gating, §4); the last H give one beta per token and head:
        alpha[b][h] = sigmoid(mean_t (X w_gate)[b][t][h]),
        beta[b][h][t] = sigmoid((X w_gate)[b][t][H + h])."""
    G = _f64(X) @ _f64(w_gate)
    sig = lambda z: 1.0 / (1.0 + np.exp(-z))
    alpha = sig(G[..., :heads].mean(axis=1))
    beta = np.transpose(sig(G[..., heads:]), (0, 2, 1))
    return alpha, beta


def block_query(S, X, weights, phi, scale=None):
    """A denoising step of the block: Y = frame_query(Q, K, V) W_o."""
    w_qkv, w_o, _ = weights
    H = phi[0].shape[0]
    Q, K, V = block_projections(X, w_qkv, H)
    O = frame_query(S, Q, K, V, phi, scale)
    B, L = O.shape[:2]
    return O.reshape(B, L, -1) @ _f64(w_o)


def block_commit(S, X, weights, phi, corr_scale=1.0, scale=None):
    """The clean pass of the block: gates from X, the layer's commit, Y = O W_o.
    Returns (Y [B, L, D], S_N)."""
    w_qkv, w_o, w_gate = weights
    H = phi[0].shape[0]
    Q, K, V = block_projections(X, w_qkv, H)
    alpha, beta = block_gates(X, w_gate, H)
    O, S_new = frame_commit(S, Q, K, V, phi, alpha, beta, corr_scale, scale)
    B, L = O.shape[:2]
    return O.reshape(B, L, -1) @ _f64(w_o), S_new
