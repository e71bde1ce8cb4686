"""Pins for the oracle's input preparation (CPU only): closed values and identities of
softplus, sigmoid and the L2 normalisation, checked so that a dropped term, a wrong sign or a
wrong axis fails at least one of them (mutation tests at the end)."""
import math

import numpy as np
import pytest

from oracle import input_prep as ip

GRID = np.array([-745.0, -700.0, -50.0, -20.0, -3.5, -1.0, -1e-8, 0.0, 1e-8, 0.25, 1.0, 3.5, 20.0, 50.0, 700.0])


def pins_softplus(softplus):
    # closed values: softplus(0) = ln 2, softplus(1) = ln(1 + e), softplus(-1) = ln(1 + 1/e)
    assert abs(softplus(np.array(0.0)) - math.log(2.0)) < 1e-15
    assert abs(softplus(np.array(1.0)) - 1.3132616875182228) < 1e-15
    assert abs(softplus(np.array(-1.0)) - 0.31326168751822286) < 1e-15
    # identity softplus(a) - softplus(-a) = a, bounds max(a, 0) <= softplus(a) <= max(a, 0) + ln 2
    sp, sn = softplus(GRID), softplus(-GRID)
    assert np.all(np.isfinite(sp))
    assert np.allclose(sp - sn, GRID, rtol=1e-15, atol=1e-13)
    assert np.all(sp >= np.maximum(GRID, 0.0)) and np.all(sp <= np.maximum(GRID, 0.0) + math.log(2.0) + 1e-15)
    # large a: softplus(a) = a + exp(-a) (first order); very negative a: exp(a)
    assert abs(softplus(np.array(40.0)) - 40.0) < 1e-15
    assert abs(softplus(np.array(-40.0)) / math.exp(-40.0) - 1.0) < 1e-12


def pins_sigmoid(sigmoid):
    assert sigmoid(np.array(0.0)) == 0.5
    assert abs(sigmoid(np.array(2.0)) - 0.8807970779778823) < 1e-15
    s, t = sigmoid(GRID), sigmoid(-GRID)
    assert np.all((s >= 0.0) & (s <= 1.0))
    assert np.allclose(s + t, 1.0, rtol=0, atol=1e-15)
    assert np.all(np.diff(sigmoid(np.sort(GRID))) >= 0.0)


def pins_decay(softplus, sigmoid):
    # alpha = exp(-softplus(a)) = 1 / (1 + e^a) = sigmoid(-a): the decay lies in (0, 1)
    alpha = np.exp(-softplus(GRID))
    assert np.allclose(alpha, sigmoid(-GRID), rtol=1e-14, atol=1e-300)
    assert np.all((alpha >= 0.0) & (alpha <= 1.0))
    assert abs(np.exp(-softplus(np.array(0.0))) - 0.5) < 1e-16


def pins_normalise(normalise):
    assert np.allclose(normalise(np.array([[3.0, 4.0]])), [[0.6, 0.8]], rtol=0, atol=1e-16)
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, 3, 16))
    xh = normalise(x)
    assert np.allclose(np.linalg.norm(xh, axis=-1), 1.0, atol=1e-15)
    # same direction: x_hat . x = ||x||; invariant to a positive scale
    assert np.allclose(np.sum(xh * x, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-14)
    assert np.allclose(normalise(7.5 * x), xh, atol=1e-15)
    # the zero vector stays zero; a vector below eps in norm is divided by eps
    assert np.array_equal(normalise(np.zeros((1, 4))), np.zeros((1, 4)))
    tiny = np.array([[1e-14, 0.0, 0.0]])
    assert np.allclose(normalise(tiny), tiny / 1e-12, rtol=1e-15)


def test_pins_accept_the_oracle():
    pins_softplus(ip.softplus)
    pins_sigmoid(ip.sigmoid)
    pins_decay(ip.softplus, ip.sigmoid)
    pins_normalise(ip.l2_normalise)


def test_prep_inputs_composes_the_steps():
    rng = np.random.default_rng(8)
    q, k = rng.standard_normal((6, 2, 8)), rng.standard_normal((6, 2, 8))
    a, b = rng.standard_normal((6, 2)), rng.standard_normal((6, 2))
    qh, kh, g, beta = ip.prep_inputs(q, k, a, b)
    assert np.allclose(np.linalg.norm(qh, axis=-1), 1.0) and np.allclose(np.linalg.norm(kh, axis=-1), 1.0)
    assert np.all(g <= 0.0) and np.allclose(np.exp(g), 1.0 / (1.0 + np.exp(a)))
    assert np.all((beta > 0.0) & (beta < 1.0)) and np.allclose(beta, 1.0 / (1.0 + np.exp(-b)))


MUTANTS = {
    "softplus without the max(a, 0) term": dict(softplus=lambda a: np.log1p(np.exp(-np.abs(ip.as_f64(a))))),
    "softplus with exp(+|a|)": dict(softplus=lambda a: np.maximum(ip.as_f64(a), 0) + np.log1p(np.exp(np.abs(ip.as_f64(a))))),
    "sigmoid of +b in the exponent": dict(sigmoid=lambda b: 1.0 / (1.0 + np.exp(ip.as_f64(b)))),
    "normalise over the wrong axis": dict(normalise=lambda x: ip.as_f64(x) / np.maximum(
        np.sqrt(np.sum(ip.as_f64(x) ** 2, axis=0, keepdims=True)), 1e-12)),
    "normalise by the squared norm": dict(normalise=lambda x: ip.as_f64(x) / np.maximum(
        np.sum(ip.as_f64(x) ** 2, axis=-1, keepdims=True), 1e-12)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistakes(name):
    m = MUTANTS[name]
    sp, sg, nm = m.get("softplus", ip.softplus), m.get("sigmoid", ip.sigmoid), m.get("normalise", ip.l2_normalise)
    with pytest.raises(AssertionError):
        pins_softplus(sp)
        pins_sigmoid(sg)
        pins_decay(sp, sg)
        pins_normalise(nm)
