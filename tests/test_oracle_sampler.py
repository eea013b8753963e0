"""Pins of the oracle's sampler pieces: sigma schedule, CFG combine, Euler step."""
import numpy as np
import pytest

import oracle as O


def test_schedule_endpoints_and_shape():
    s = O.sigma_schedule(25, 1.73)
    assert s.shape == (26,)
    assert s[0] == pytest.approx(1.0, abs=1e-15)
    assert s[-1] == 0.0
    assert np.all(np.diff(s) < 0)


def test_schedule_unshifted_is_linspace():
    s = O.sigma_schedule(10, 1.0)
    assert np.allclose(s[:-1], np.linspace(1.0, 0.001, 10), atol=1e-15)


def test_schedule_closed_form_value():
    k = 1.73
    base = 1.0 - 0.999 / 24.0
    expect = k * base / (1.0 + (k - 1.0) * base)
    assert O.sigma_schedule(25, k)[1] == pytest.approx(expect, rel=1e-14)
    # a shift above 1 spends more of the schedule at high noise
    assert np.all(O.sigma_schedule(25, k)[1:-1] > O.sigma_schedule(25, 1.0)[1:-1])


def test_euler_noop_when_sigma_unchanged():
    rng = np.random.default_rng(0)
    x, v = rng.standard_normal((1, 4, 8, 8)), rng.standard_normal((2, 4, 8, 8))
    assert np.array_equal(O.euler_cfg_step(x, v, 3.5, 0.6, 0.6), x)


def test_cfg_special_cases():
    rng = np.random.default_rng(1)
    vu, vc = rng.standard_normal((3, 5)), rng.standard_normal((3, 5))
    assert np.allclose(O.cfg_combine(vu, vc, 1.0), vc, atol=1e-15)
    assert np.array_equal(O.cfg_combine(vu, vc, 0.0), vu)
    assert np.allclose(O.cfg_combine(vu, vc, 3.5), 3.5 * vc - 2.5 * vu, atol=1e-14)


def test_euler_straight_line_exactness():
    """x_sigma = (1 - sigma) x0 + sigma eps with v = eps - x0 lands on x_sigma'."""
    rng = np.random.default_rng(2)
    x0, eps = rng.standard_normal((1, 4, 6, 6)), rng.standard_normal((1, 4, 6, 6))
    s, s2 = 0.83, 0.41
    xs = (1 - s) * x0 + s * eps
    v = np.concatenate([eps - x0, eps - x0])     # identical halves: CFG is a no-op
    out = O.euler_cfg_step(xs, v, 3.5, s, s2)
    assert np.allclose(out, (1 - s2) * x0 + s2 * eps, atol=1e-14)
    # stepping all the way to sigma = 0 recovers x0
    assert np.allclose(O.euler_cfg_step(xs, v, 3.5, s, 0.0), x0, atol=1e-14)


def test_cfg_uses_uncond_first():
    x = np.zeros((1, 1, 2, 2))
    v = np.concatenate([np.full((1, 1, 2, 2), 1.0), np.full((1, 1, 2, 2), 3.0)])
    # g = 2: v = 1 + 2 (3 - 1) = 5 ; step -0.1 -> -0.5
    assert np.allclose(O.euler_cfg_step(x, v, 2.0, 0.5, 0.4), -0.5, atol=1e-15)
