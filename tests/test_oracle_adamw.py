"""Pins of the oracle's AdamW step (teardown section 5, paged AdamW; the update is AdamW with
decoupled weight decay)."""

from fractions import Fraction

import numpy as np

from oracle import adamw


def test_first_step_from_zero_states():
    rng = np.random.default_rng(0)
    g = rng.standard_normal(1000)
    p0 = rng.standard_normal(1000)
    lr, eps = 1e-3, 1e-8
    p, m, v = adamw.adamw_step(p0, g, np.zeros(1000), np.zeros(1000), lr, 0.9, 0.999, eps, 0.0, 1)
    assert np.allclose(p, p0 - lr * g / (np.abs(g) + eps), rtol=0, atol=1e-15)
    assert np.allclose(m, 0.1 * g) and np.allclose(v, 0.001 * g * g)


def test_zero_gradient_only_decays():
    p0 = np.linspace(-1, 1, 11)
    p, m, v = adamw.adamw_step(p0, np.zeros(11), np.zeros(11), np.zeros(11), 0.01, 0.9, 0.999, 1e-8, 0.1, 3)
    assert np.allclose(p, p0 * (1 - 0.01 * 0.1), rtol=0, atol=1e-16)
    assert np.all(m == 0) and np.all(v == 0)


def test_two_steps_against_exact_rationals():
    # beta2 = 3/4 keeps every v-hat a perfect square here, so the square root is exact
    b1, b2, lr, wd = Fraction(1, 2), Fraction(3, 4), Fraction(1, 8), Fraction(1, 4)
    p, m, v = Fraction(1), Fraction(0), Fraction(0)
    for t, g in ((1, Fraction(2)), (2, Fraction(2))):
        m = b1 * m + (1 - b1) * g
        v = b2 * v + (1 - b2) * g * g
        mhat, vhat = m / (1 - b1 ** t), v / (1 - b2 ** t)
        root = Fraction(int(round(float(vhat) ** 0.5)))
        assert root * root == vhat
        p = p - lr * (mhat / root + wd * p)
    pf, mf, vf = 1.0, 0.0, 0.0
    for t in (1, 2):
        pf, mf, vf = adamw.adamw_step(pf, 2.0, mf, vf, 0.125, 0.5, 0.75, 0.0, 0.25, t)
    assert float(pf) == float(p) and float(mf) == float(m) and float(vf) == float(v)
