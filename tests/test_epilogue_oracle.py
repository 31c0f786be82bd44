"""Pins of the output epilogue's oracle (gated RMS normalisation over each
head's value channels) against facts that do not come from the oracle itself:
the library RMS normalisation, closed forms of the logistic function, scale
invariance, unit RMS and a hand-worked case.  The last test plants plausible
mistakes in copies of the oracle function and requires a pin to catch each."""
import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import epilogue

D = 128


def _case(seed, shape=(5, 3), eps=1e-5):
    rng = np.random.default_rng(seed)
    scale = np.exp(rng.normal(0.0, 2.0, size=shape + (1,)))  # per (token, head) scales
    o = rng.normal(size=shape + (D,)) * scale
    z = rng.normal(0.0, 3.0, size=shape + (D,))
    w = rng.uniform(0.2, 2.0, size=D)
    return o, z, w, eps


def pin_library_rmsnorm(f):
    """With the gate saturated (sigmoid = 1 in fp64) the epilogue is the
    library's RMS normalisation with weight w over the last axis."""
    o, _, w, eps = _case(1)
    z = np.full(o.shape, 60.0)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(o), (D,), torch.from_numpy(w), eps).numpy()
    np.testing.assert_allclose(f(o, z, w, eps), ref, rtol=1e-12, atol=0)


def pin_scale_invariance(f):
    """At eps = 0 the output of a (token, head) does not depend on its scale."""
    o, z, w, _ = _case(2)
    c = np.exp(np.random.default_rng(3).normal(0, 3, size=o.shape[:-1] + (1,)))
    np.testing.assert_allclose(f(o * c, z, w, 0.0), f(o, z, w, 0.0), rtol=1e-12, atol=0)


def pin_unit_rms(f):
    """At eps = 0, y / (w sigmoid(z)) has RMS 1 over each head's channels."""
    o, z, w, _ = _case(4)
    y = f(o, z, w, 0.0) / (w * scipy.special.expit(z))
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-12)


def pin_gate_closed_forms(f):
    """z = 0 halves the normalised output; z and -z gates add up to the ungated
    output (sigmoid(z) + sigmoid(-z) = 1); the gate is the library logistic."""
    o, z, w, eps = _case(5)
    full = f(o, np.full(o.shape, 60.0), w, eps)
    np.testing.assert_allclose(f(o, np.zeros(o.shape), w, eps), 0.5 * full, rtol=1e-14)
    np.testing.assert_allclose(f(o, z, w, eps) + f(o, -z, w, eps), full, rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(f(o, z, w, eps), full * scipy.special.expit(z), rtol=1e-12)


def pin_hand_worked(f):
    """d = 2, o = (3, 4), eps = 0: RMS = sqrt(12.5) = 5/sqrt(2), so with w = (1, 2)
    and gates (0, +inf) the output is (0.5 * 3, 2 * 4) * sqrt(2) / 5."""
    y = f(np.array([3.0, 4.0]), np.array([0.0, 800.0]), np.array([1.0, 2.0]), 0.0)
    np.testing.assert_allclose(y, np.array([1.5, 8.0]) * np.sqrt(2.0) / 5.0, rtol=1e-15)


def pin_eps_inside_root(f):
    """eps enters under the square root: o = (e, e), eps = 3 e^2 gives RMS 2 e."""
    e = 1e-3
    y = f(np.array([e, e]), np.array([800.0, 800.0]), np.ones(2), 3 * e * e)
    np.testing.assert_allclose(y, [0.5, 0.5], rtol=1e-14)


PINS = [pin_library_rmsnorm, pin_scale_invariance, pin_unit_rms, pin_gate_closed_forms,
        pin_hand_worked, pin_eps_inside_root]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle.epilogue.gated_rmsnorm)


def test_sigmoid_extremes():
    z = np.array([-800.0, -40.0, 0.0, 40.0, 800.0])
    s = epilogue.sigmoid(z)
    assert np.all(np.isfinite(s))
    np.testing.assert_allclose(s, scipy.special.expit(z), rtol=1e-15, atol=0)


def _mean_sq(o):
    return np.mean(o * o, axis=-1, keepdims=True)


MUTANTS = {
    "sum instead of mean": lambda o, z, w, e: o / np.sqrt(np.sum(o * o, -1, keepdims=True) + e) * w * epilogue.sigmoid(z),
    "eps outside the root": lambda o, z, w, e: o / (np.sqrt(_mean_sq(o)) + e) * w * epilogue.sigmoid(z),
    "weight dropped": lambda o, z, w, e: o / np.sqrt(_mean_sq(o) + e) * epilogue.sigmoid(z),
    "gate of -z": lambda o, z, w, e: o / np.sqrt(_mean_sq(o) + e) * w * epilogue.sigmoid(-z),
    "gate not applied": lambda o, z, w, e: o / np.sqrt(_mean_sq(o) + e) * w,
    "norm over the wrong axis": lambda o, z, w, e: o / np.sqrt(np.mean(o * o, 0, keepdims=True) + e) * w * epilogue.sigmoid(z),
    "rms without the root": lambda o, z, w, e: o / (_mean_sq(o) + e) * w * epilogue.sigmoid(z),
    "gate exp(z)": lambda o, z, w, e: o / np.sqrt(_mean_sq(o) + e) * w * np.exp(np.minimum(z, 700)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    f = MUTANTS[name]
    caught = 0
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(f)
        except (AssertionError, ValueError):
            caught += 1
    assert caught > 0, f"no pin catches: {name}"
