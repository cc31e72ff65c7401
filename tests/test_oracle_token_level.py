"""The oracle's token-level pass against its pins, and planted mistakes in
copies of it that the pins must catch (a state read after the write, a
prediction from the decayed state, a transposed outer product, a dropped
gate or coefficient, unnormalised keys)."""
import types

import numpy as np
import pytest

from oracle import arl2_oracle as real
from tests.oracle_token_pins import TOKEN_PINS

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


@pytest.mark.parametrize("pin", TOKEN_PINS, ids=lambda f: f.__name__)
def test_token_pin(pin):
    pin(real)


def _scan(S, Q, K, V, phi, a, beta, c, scale=None, *, after_write=False, decayed_pred=False,
          transposed=False, no_beta=False, no_c=False, no_norm=False, decay_delta=False):
    """A token-level pass with one planted mistake switched on."""
    St = np.array(S, dtype=np.float64)
    Qp, Kp, Vp = real.feature_maps(Q, K, V, *phi)
    if no_norm:
        Kp = np.asarray(K, dtype=np.float64).transpose(0, 2, 1, 3) @ np.asarray(phi[1])[None]
    a, beta = np.asarray(a, dtype=np.float64), np.asarray(beta, dtype=np.float64)
    c = 1.0 if no_c else float(c)
    B, H, L, _ = Qp.shape
    Oi = np.empty((B, H, L, St.shape[-1]))
    for t in range(L):
        if not after_write:
            Oi[:, :, t] = np.einsum("bhi,bhij->bhj", Qp[:, :, t], St)
        base = a[:, :, t, None, None] * St if decayed_pred else St
        pred = np.einsum("bhi,bhij->bhj", Kp[:, :, t], base)
        r = (1.0 if no_beta else beta[:, :, t, None]) * (Vp[:, :, t] - pred)
        outer = Kp[:, :, t, :, None] * r[:, :, None, :]
        if transposed:
            outer = np.swapaxes(outer, -1, -2)
        if decay_delta:
            St = a[:, :, t, None, None] * (St + c * outer)
        else:
            St = a[:, :, t, None, None] * St + c * outer
        if after_write:
            Oi[:, :, t] = np.einsum("bhi,bhij->bhj", Qp[:, :, t], St)
    O = real.intra_softmax(Q, K, V, scale) + np.ascontiguousarray(Oi.transpose(0, 2, 1, 3))
    return O, St


MUTANTS = ["after_write", "decayed_pred", "transposed", "no_beta", "no_c", "no_norm", "decay_delta"]


def _mutant(flag):
    ns = types.SimpleNamespace(**{k: getattr(real, k) for k in real.__all__})
    ns.token_level_pass = lambda *args, **kw: _scan(*args, **kw, **{flag: True})
    return ns


def test_unmutated_copy_passes_every_pin():
    ns = types.SimpleNamespace(**{k: getattr(real, k) for k in real.__all__})
    ns.token_level_pass = lambda *args, **kw: _scan(*args, **kw)
    for pin in TOKEN_PINS:
        pin(ns)


@pytest.mark.parametrize("flag", MUTANTS)
def test_pins_catch_mutant(flag):
    failed = []
    for pin in TOKEN_PINS:
        try:
            pin(_mutant(flag))
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin catches the mutant {flag}"
