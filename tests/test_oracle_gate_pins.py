"""Pins for the oracle's gate activation from raw projections (g = -a softplus(x + b),
beta = sigmoid(y), per V head), independent of the oracle's own code: exact values of
softplus and sigmoid, their inverses in closed form, the identities that tie them
together, their limits, and the per-head wiring into the recurrence.
"""

import math

import numpy as np
import pytest

import oracle


def test_exact_values():
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    assert oracle.sigmoid(0.0) == 0.5
    assert oracle.sigmoid(math.log(3.0)) == pytest.approx(0.75, rel=1e-15)  # 1 / (1 + 1/3)
    assert oracle.softplus(math.log(math.e - 1.0)) == pytest.approx(1.0, rel=1e-15)


@pytest.mark.parametrize("c", [1e-8, 1e-3, 0.5, 2.0, 30.0])
def test_softplus_inverts_in_closed_form(c):
    # softplus(z) = c  <=>  z = log(exp(c) - 1) = c + log(1 - exp(-c))
    z = c + math.log(-math.expm1(-c))
    assert oracle.softplus(z) == pytest.approx(c, rel=1e-12)


def test_identities_and_limits():
    z = np.linspace(-40, 40, 801)
    np.testing.assert_allclose(oracle.softplus(z) - oracle.softplus(-z), z, rtol=0, atol=1e-13)
    np.testing.assert_allclose(oracle.sigmoid(z) + oracle.sigmoid(-z), 1.0, rtol=0, atol=1e-15)
    # d softplus / dz = sigmoid (central differences, step 1e-5)
    h = 1e-5
    fd = (oracle.softplus(z + h) - oracle.softplus(z - h)) / (2 * h)
    np.testing.assert_allclose(fd, oracle.sigmoid(z), rtol=0, atol=1e-9)
    # log sigmoid(y) = -softplus(-y)
    np.testing.assert_allclose(np.log(oracle.sigmoid(z)), -oracle.softplus(-z), rtol=1e-12, atol=1e-15)
    assert oracle.softplus(800.0) == 800.0 and oracle.softplus(-800.0) == 0.0
    assert oracle.sigmoid(800.0) == 1.0 and oracle.sigmoid(-800.0) == 0.0


def _per_head_inputs(seed, T=5, HV=6):
    r = np.random.default_rng(seed)
    a = r.uniform(0.1, 8.0, HV)       # per-head decay rate
    b = r.normal(0.0, 2.0, HV)        # per-head bias
    c = r.uniform(0.01, 3.0, (T, HV))  # wanted softplus values
    p = r.uniform(0.02, 0.98, (T, HV))  # wanted beta values
    x = c + np.log(-np.expm1(-c)) - b[None, :]
    y = np.log(p / (1.0 - p))
    return a, b, c, p, x, y


def test_per_head_wiring():
    a, b, c, p, x, y = _per_head_inputs(0)
    g, beta = oracle.gates_from_projections(x, y, a, b)
    np.testing.assert_allclose(g, -a[None, :] * c, rtol=1e-12)
    np.testing.assert_allclose(beta, p, rtol=1e-12)
    assert np.all(g < 0) and np.all((beta > 0) & (beta < 1))


def test_forward_from_projections_uses_the_activated_gates():
    a, b, c, p, x, y = _per_head_inputs(1, T=9, HV=4)
    r = np.random.default_rng(2)
    q, k = r.standard_normal((9, 2, 16)), r.standard_normal((9, 2, 16))
    v = r.standard_normal((9, 4, 8))
    s0 = r.standard_normal((2, 4, 8, 16))
    cu = [0, 4, 9]
    out_p, fin_p = oracle.forward_from_projections(q, k, v, x, y, a, b, cu, s0)
    out, fin = oracle.forward(q, k, v, -a[None, :] * c, p, cu, s0)
    np.testing.assert_allclose(out_p, out, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(fin_p, fin, rtol=1e-11, atol=1e-13)
    # decode form: the same tokens as [N=1, ntok, ...] continued from a state
    o_d, s_d = oracle.decode_from_projections(q[None, :4], k[None, :4], v[None, :4], x[None, :4], y[None, :4],
                                              a, b, s0[:1])
    np.testing.assert_allclose(o_d[0], out[:4], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(s_d[0], fin[0], rtol=1e-11, atol=1e-13)


# Plausible slips in the activation; each must fail the wiring pin.
def _bias_outside(x, y, a, b):
    return -a[None, :] * (oracle.softplus(x) + b[None, :]), oracle.sigmoid(y)


def _rate_as_log(x, y, a, b):
    return -np.exp(a)[None, :] * oracle.softplus(x + b[None, :]), oracle.sigmoid(y)


def _sigmoid_sign(x, y, a, b):
    return -a[None, :] * oracle.softplus(x + b[None, :]), oracle.sigmoid(-y)


def _bias_transposed(x, y, a, b):
    return -a[None, :] * oracle.softplus(x + b[::-1][None, :]), oracle.sigmoid(y)


@pytest.mark.parametrize("mutant", [_bias_outside, _rate_as_log, _sigmoid_sign, _bias_transposed])
def test_pins_reject_planted_mistakes(mutant):
    a, b, c, p, x, y = _per_head_inputs(3)
    g, beta = mutant(x, y, a, b)
    ok = np.allclose(g, -a[None, :] * c, rtol=1e-9) and np.allclose(beta, p, rtol=1e-9)
    assert not ok
