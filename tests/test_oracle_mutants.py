"""Planted mistakes in the oracle must be caught by its pins.

Each mutant is a copy of the oracle with one plausible error (a dropped
term, a transposed operand, a wrong axis, a state read after the write).
The test passes when at least one pin fails on the mutant; the real oracle
passing every pin is checked in test_oracle_pins.py.
"""
import types

import numpy as np
import pytest

from oracle import arl2_oracle as real
from tests.oracle_pins import ALL_PINS


def _clone(**overrides):
    ns = types.SimpleNamespace(**{k: getattr(real, k) for k in real.__all__})
    for k, v in overrides.items():
        setattr(ns, k, v)
    # rebind the composite functions so that they call the overridden pieces
    fm, intra, ro = ns.feature_maps, ns.intra_softmax, ns.inter_readout

    def frame_query(S, Q, K, V, phi, scale=None):
        Qp, _, _ = fm(Q, K, V, *phi)
        return intra(Q, K, V, scale) + ro(Qp, S)

    if "frame_query" not in overrides:
        ns.frame_query = frame_query
    fq = ns.frame_query

    def frame_commit(S, Q, K, V, phi, alpha, beta, corr_scale=1.0, scale=None):
        S = np.asarray(S, dtype=np.float64)
        O = fq(S, Q, K, V, phi, scale)
        _, Kp, Vp = fm(Q, K, V, *phi)
        R = np.asarray(beta)[..., None] * (Vp - Kp @ S)
        delta = np.swapaxes(Kp, -1, -2) @ R
        return O, np.asarray(alpha)[..., None, None] * S + corr_scale * delta

    if "frame_commit" not in overrides:
        ns.frame_commit = frame_commit
    ns.kv_attention = lambda Q, K, V, scale=None: ns.intra_softmax(Q, K, V, scale)
    return ns


def _fm_transposed_phi(Q, K, V, pq, pk, pv):
    t = lambda p: np.swapaxes(np.asarray(p, dtype=np.float64), -1, -2)
    return real.feature_maps(Q, K, V, t(pq), t(pk), t(pv))


def _fm_no_norm(Q, K, V, pq, pk, pv):
    Qh, Kh, Vh = (np.asarray(x, dtype=np.float64).transpose(0, 2, 1, 3) for x in (Q, K, V))
    return Qh @ pq[None], Kh @ pk[None], Vh @ pv[None]


def _intra_no_scale(Q, K, V, scale=None):
    return real.intra_softmax(Q, K, V, 1.0)


def _intra_wrong_max_axis(Q, K, V, scale=None):
    Qh, Kh, Vh = (np.asarray(x, dtype=np.float64).transpose(0, 2, 1, 3) for x in (Q, K, V))
    s = (Qh @ np.swapaxes(Kh, -1, -2)) * Qh.shape[-1] ** -0.5
    p = np.exp(s - s.max(axis=-2, keepdims=True))
    return ((p @ Vh) / p.sum(axis=-2, keepdims=True)).transpose(0, 2, 1, 3)


def _readout_transposed_state(Qp, S):
    return real.inter_readout(Qp, np.swapaxes(np.asarray(S, dtype=np.float64), -1, -2))


def _commit(variant):
    def frame_commit(S, Q, K, V, phi, alpha, beta, corr_scale=1.0, scale=None):
        S = np.asarray(S, dtype=np.float64)
        _, Kp, Vp = real.feature_maps(Q, K, V, *phi)
        a = np.asarray(alpha)[..., None, None]
        b = np.asarray(beta)[..., None]
        if variant == "no_beta":
            R = Vp - Kp @ S
        elif variant == "no_prediction":
            R = b * Vp
        else:
            R = b * (Vp - Kp @ S)
        delta = np.swapaxes(Kp, -1, -2) @ R
        if variant == "delta_transposed":
            delta = np.swapaxes(delta, -1, -2)
        if variant == "decay_inside":
            S_new = a * (S + corr_scale * delta)
        else:
            S_new = a * S + corr_scale * delta
        O = real.frame_query(S_new if variant == "read_after_write" else S, Q, K, V, phi, scale)
        return O, S_new
    return frame_commit


MUTANTS = {
    "phi_transposed": _clone(feature_maps=_fm_transposed_phi),
    "key_not_normalised": _clone(feature_maps=_fm_no_norm),
    "softmax_unscaled": _clone(intra_softmax=_intra_no_scale),
    "softmax_max_wrong_axis": _clone(intra_softmax=_intra_wrong_max_axis),
    "readout_state_transposed": _clone(inter_readout=_readout_transposed_state),
    "update_without_beta": _clone(frame_commit=_commit("no_beta")),
    "update_without_prediction": _clone(frame_commit=_commit("no_prediction")),
    "update_delta_transposed": _clone(frame_commit=_commit("delta_transposed")),
    "update_decay_inside": _clone(frame_commit=_commit("decay_inside")),
    "readout_after_write": _clone(frame_commit=_commit("read_after_write")),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    mutant = MUTANTS[name]
    failed = []
    for pin in ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin catches the mutant {name}"
