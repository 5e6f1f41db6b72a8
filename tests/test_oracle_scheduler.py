"""Pins of the oracle's FlowMatch-Euler schedule, update and CFG combine."""
from fractions import Fraction

import numpy as np
import pytest

from conftest import read_golden
from oracle import scheduler_ref as sch


def test_sigmas_match_exact_fractions():
    rows = read_golden("sigmas_shift3_n8.txt")
    want = [float(Fraction(int(n), int(d))) for _, n, d in rows]
    got = sch.sigmas(8, 3.0)
    assert len(got) == 9
    np.testing.assert_allclose(got, want, rtol=1e-15, atol=0)


def test_shift_closed_forms():
    assert sch.shift_sigma(0.5, 3.0) == pytest.approx(0.75, rel=1e-15)
    s = np.linspace(0, 1, 11)
    np.testing.assert_allclose(sch.shift_sigma(s, 1.0), s, rtol=1e-15)
    sig = sch.sigmas(8)
    assert np.all(np.diff(sig) < 0)
    assert sig[0] == 1.0 and sig[-1] == 0.0
    # the Euler step sizes telescope to -1
    assert np.sum(np.diff(sig)) == pytest.approx(-1.0, abs=1e-15)


def test_timesteps_are_one_minus_sigma():
    sig = sch.sigmas(8)
    t = sch.timesteps(sig)
    assert len(t) == 8  # the zero-sigma call is skipped
    np.testing.assert_allclose(t, 1.0 - sig[:-1], rtol=0, atol=0)
    assert t[0] == 0.0  # pure noise at t = 0, 1 = clean


def test_constant_velocity_telescopes():
    """A model that always outputs y makes x_N = x_0 + y (v = -y, sum of steps = -1)."""
    rng = np.random.default_rng(0)
    x0 = rng.standard_normal((1, 16, 4, 4))
    y = rng.standard_normal((1, 16, 4, 4))
    xN = sch.denoise(x0, lambda x, t, u: y, 8, 3.0)
    np.testing.assert_allclose(xN, x0 + y, rtol=1e-13, atol=1e-13)


def test_model_sees_the_shifted_timesteps():
    seen = []
    sch.denoise(np.zeros((2, 1, 2, 2)), lambda x, t, u: (seen.append(t.copy()), np.zeros_like(x))[1], 8)
    np.testing.assert_allclose(np.array(seen)[:, 0], sch.timesteps(sch.sigmas(8)), rtol=1e-15)


def test_euler_step_sign():
    # model output +1 at sigma 1 -> 0.5 moves x by +0.5 (velocity -1, dt = -0.5)
    assert sch.euler_step(np.array([0.0]), np.array([1.0]), 1.0, 0.5)[0] == 0.5


def test_cfg_combine_special_cases():
    rng = np.random.default_rng(1)
    yc, yu = rng.standard_normal(5), rng.standard_normal(5)
    np.testing.assert_allclose(sch.cfg_combine(yc, yu, 1.0), yc, rtol=0, atol=1e-15)
    np.testing.assert_array_equal(sch.cfg_combine(yc, yu, 0.0), yu)
    # guidance 4 equals the pipeline form y_c + 3 (y_c - y_u) (ai-toolkit: UI 4 -> pipeline 3)
    np.testing.assert_allclose(sch.cfg_combine(yc, yu, 4.0), yc + 3.0 * (yc - yu), rtol=1e-14)
