"""Pins for the oracle's design-time codebook (AXELRAM Abstract: the optimal quantizer for N(0,1/d) depends only
on d and b).  Checked against closed forms, a printed table, and optimality conditions evaluated with an independent
numerical integrator (scipy.integrate.quad), not with the oracle's own formulas."""

import math
import os

import numpy as np
import pytest
from scipy import integrate

import oracle

HERE = os.path.dirname(__file__)


def _golden():
    rows = {}
    with open(os.path.join(HERE, "golden", "lloyd_max_gaussian.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            rows[(int(parts[0]), parts[1])] = [float(x) for x in parts[2:]]
    return rows


def _pdf(x):
    return math.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)


def _quad(f, a, b):
    val, err = integrate.quad(f, a, b, epsabs=1e-14, epsrel=1e-13, limit=200)
    return val


def _distortion(levels, thresholds):
    edges = [-np.inf] + list(thresholds) + [np.inf]
    return sum(_quad(lambda x, c=c: (x - c) ** 2 * _pdf(x), edges[k], edges[k + 1]) for k, c in enumerate(levels))


def test_one_bit_closed_form():
    g, t = oracle.gaussian_lloyd_max(1)
    r = math.sqrt(2 / math.pi)
    assert np.allclose(g, [-r, r], rtol=0, atol=1e-14)
    assert np.allclose(t, [0.0], atol=1e-15)
    assert abs(_distortion(g, t) - (1 - 2 / math.pi)) < 1e-12


@pytest.mark.parametrize("bits", [1, 2])
def test_printed_table(bits):
    gold = _golden()
    g, t = oracle.gaussian_lloyd_max(bits)
    L = 1 << bits
    lv = gold[(bits, "levels")]
    th = gold[(bits, "thresholds")]
    # values printed to 4 significant figures: compare at half a unit of the last printed digit
    for got, want in zip(g[L // 2:], lv):
        digits = 4 - 1 - int(math.floor(math.log10(abs(want))))
        assert abs(got - want) <= 0.5 * 10 ** (-digits) + 1e-12, (got, want)
    for got, want in zip(t[L // 2 - 1:], th):
        if want == 0:
            assert abs(got) < 1e-15
        else:
            digits = 4 - 1 - int(math.floor(math.log10(abs(want))))
            assert abs(got - want) <= 0.5 * 10 ** (-digits) + 1e-12
    mse = gold[(bits, "mse")][0]
    D = _distortion(g, t)
    if bits == 1:
        assert abs(D - mse) < 1e-12
    else:
        assert abs(D - mse) <= 0.5e-4


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_optimality_conditions_by_quadrature(bits):
    """Lloyd-Max necessary conditions, evaluated by numerical integration:
    each level is the conditional mean of its cell, each threshold the midpoint of its neighbours."""
    g, t = oracle.gaussian_lloyd_max(bits)
    edges = [-np.inf] + list(t) + [np.inf]
    for k in range(len(g)):
        mass = _quad(_pdf, edges[k], edges[k + 1])
        mean = _quad(lambda x: x * _pdf(x), edges[k], edges[k + 1]) / mass
        assert abs(mean - g[k]) < 1e-10, (bits, k, mean, g[k])
    for k in range(1, len(g)):
        assert abs(t[k - 1] - 0.5 * (g[k - 1] + g[k])) < 1e-15


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_local_minimum_of_distortion(bits):
    """Moving any single level by +-1e-3 (thresholds re-optimised as midpoints) raises the distortion."""
    g, t = oracle.gaussian_lloyd_max(bits)
    D0 = _distortion(g, t)
    for k in range(len(g)):
        for eps in (-1e-3, 1e-3):
            g2 = g.copy()
            g2[k] += eps
            t2 = 0.5 * (g2[:-1] + g2[1:])
            assert _distortion(g2, t2) > D0


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_symmetry_and_order(bits):
    g, t = oracle.gaussian_lloyd_max(bits)
    assert np.all(np.diff(g) > 0) and np.all(np.diff(t) > 0)
    assert np.allclose(g, -g[::-1], atol=1e-14)
    assert np.allclose(t, -t[::-1], atol=1e-14)
    assert abs(t[len(t) // 2]) < 1e-15  # the middle threshold is zero


def test_distortion_decreases_with_bits():
    D = [_distortion(*oracle.gaussian_lloyd_max(b)) for b in (1, 2, 3, 4)]
    assert all(a > b for a, b in zip(D, D[1:]))
    # each extra bit buys close to the 6 dB asymptote (ratio ~ 1/4) but never better than it
    ratios = [b / a for a, b in zip(D, D[1:])]
    assert all(0.25 < r < 0.36 for r in ratios), ratios


@pytest.mark.parametrize("d", [8, 64, 128])
def test_unit_scale(d):
    for bits in (1, 2, 3, 4):
        c, t = oracle.codebook(d, bits)
        g, tau = oracle.gaussian_lloyd_max(bits)
        assert np.allclose(c * math.sqrt(d), g, rtol=1e-15, atol=0)
        assert np.allclose(t * math.sqrt(d), tau, rtol=1e-15, atol=1e-300)
