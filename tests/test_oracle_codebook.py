"""Pins for the oracle's Lloyd-Max codebook (not the CUDA path).

Pinned against: the closed form E|X| = sqrt(2/pi) at 1 bit, the textbook
Gaussian Lloyd-Max table (tests/golden/lloyd_max_gaussian.json), Lloyd's two
optimality conditions (fixed-point residual), symmetry and the 1/sqrt(d)
scaling law.
"""

import json
import math
import os

import numpy as np
import pytest
from scipy import integrate, stats

from oracle import codebook


def _matches_printed(value: float, printed: str) -> bool:
    decimals = len(printed.split(".")[1]) if "." in printed else 0
    return abs(value - float(printed)) <= 0.5 * 10.0 ** (-decimals) + 2e-6


def test_one_bit_closed_form():
    for d in (1, 64, 128, 256):
        c, t, _ = codebook.lloyd_max_gaussian(1, d)
        expect = math.sqrt(2.0 / math.pi) / math.sqrt(d)
        assert np.allclose(c, [-expect, expect], rtol=0, atol=1e-14 / math.sqrt(d))
        assert np.allclose(t, [0.0], atol=1e-15)


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_textbook_table(golden_dir, bits):
    g = json.load(open(os.path.join(golden_dir, "lloyd_max_gaussian.json")))
    lv = g["levels"][str(bits)]
    c, t, _ = codebook.lloyd_max_gaussian(bits, 1)
    pos_c = c[len(c) // 2:]
    pos_t = t[len(t) // 2 + 1:] if len(t) > 1 else []
    assert len(pos_c) == len(lv["centroids_pos"])
    for v, p in zip(pos_c, lv["centroids_pos"]):
        assert _matches_printed(float(v), p), (v, p)
    for v, p in zip(pos_t, lv["boundaries_pos"]):
        assert _matches_printed(float(v), p), (v, p)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_fixed_point_and_symmetry(bits):
    d = 128
    c, t, _ = codebook.lloyd_max_gaussian(bits, d)
    assert len(c) == 2 ** bits and len(t) == 2 ** bits - 1
    assert np.all(np.diff(c) > 0) and np.all(np.diff(t) > 0)
    assert codebook.fixed_point_residual(c, t, d) < 1e-12
    # the symmetric law's quantizer is exactly antisymmetric, the middle
    # boundary (even level count) exactly 0
    assert np.array_equal(c, -c[::-1]) and np.array_equal(t, -t[::-1])
    assert t[len(t) // 2] == 0.0
    # boundaries lie between neighbouring centroids
    assert np.all(c[:-1] < t) and np.all(t < c[1:])


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_scaling_with_d(bits):
    c1, t1, _ = codebook.lloyd_max_gaussian(bits, 1)
    for d in (64, 128, 256):
        c, t, _ = codebook.lloyd_max_gaussian(bits, d)
        assert np.allclose(c * math.sqrt(d), c1, atol=1e-12)
        assert np.allclose(t * math.sqrt(d), t1, atol=1e-12)


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_per_coordinate_mse_matches_table(golden_dir, bits):
    """E[(X - Q(X))^2] for X ~ N(0,1), by quadrature over the cells."""
    g = json.load(open(os.path.join(golden_dir, "lloyd_max_gaussian.json")))
    c, t, _ = codebook.lloyd_max_gaussian(bits, 1)
    edges = np.concatenate(([-np.inf], t, [np.inf]))
    mse = 0.0
    for i in range(len(c)):
        val, _ = integrate.quad(lambda x, ci=c[i]: (x - ci) ** 2 * stats.norm.pdf(x),
                                edges[i], edges[i + 1], epsabs=1e-13)
        mse += val
    assert _matches_printed(mse, g["per_coordinate_mse"][str(bits)]), mse


def test_centroid_is_conditional_mean_by_quadrature():
    """The centroid formula agrees with a direct quadrature of x phi(x)."""
    c, t, _ = codebook.lloyd_max_gaussian(2, 1)
    edges = np.concatenate(([-np.inf], t, [np.inf]))
    for i in range(len(c)):
        num, _ = integrate.quad(lambda x: x * stats.norm.pdf(x), edges[i], edges[i + 1])
        den, _ = integrate.quad(stats.norm.pdf, edges[i], edges[i + 1])
        assert abs(num / den - c[i]) < 1e-9
