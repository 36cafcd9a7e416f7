"""Pins for the oracle's Lloyd-Max codebook (Method step [4] of the
"Qwen3.6-35B-A3B -- HLWQ Q5" model card: 32 centroids, N(0,1), optimal MSE).

Independent anchors: the 2-level closed form, the classical optima of
J. Max, "Quantizing for minimum distortion", IRE Trans. Inf. Theory IT-6 (1960),
Table I (4 and 8 levels), numerical integration by scipy's adaptive quadrature
(not the erfc closed forms the oracle uses), Monte Carlo, and the Panter-Dite
high-rate approximation (sqrt(3) pi / 2) / L^2.
"""
import math

import numpy as np
import pytest
from scipy import integrate

import oracle as O


def phi(z):
    return math.exp(-0.5 * z * z) / math.sqrt(2 * math.pi)


def test_two_levels_closed_form():
    r = O.lloyd_max_gaussian(2)
    c = math.sqrt(2 / math.pi)          # E[|Z|]
    assert r["centroids"][1] == pytest.approx(c, abs=1e-14)
    assert r["centroids"][0] == -r["centroids"][1]
    assert r["mse"] == pytest.approx(1 - 2 / math.pi, abs=1e-13)


def test_four_levels_max_table():
    r = O.lloyd_max_gaussian(4)
    assert r["centroids"][2:] == pytest.approx([0.4528, 1.510], abs=6e-4)
    assert r["thresholds"][2] == pytest.approx(0.9816, abs=1e-4)
    assert r["mse"] == pytest.approx(0.1175, abs=1e-4)


def test_eight_levels_max_table():
    r = O.lloyd_max_gaussian(8)
    assert r["centroids"][4:] == pytest.approx([0.2451, 0.7560, 1.344, 2.152], abs=6e-4)
    assert r["thresholds"][3:] == pytest.approx([0.0, 0.5006, 1.050, 1.748], abs=6e-4)
    assert r["mse"] == pytest.approx(0.03455, abs=1e-5)


@pytest.mark.parametrize("levels", [16, 32])
def test_lloyd_conditions_by_quadrature(levels):
    """Each centroid is the conditional mean of its cell, computed by adaptive
    quadrature of z*phi and phi (independent of the oracle's closed forms)."""
    r = O.lloyd_max_gaussian(levels)
    c, t = r["centroids"], r["thresholds"]
    edges = [-np.inf] + list(t) + [np.inf]
    for k in range(levels):
        a, b = edges[k], edges[k + 1]
        m0 = integrate.quad(phi, a, b, epsabs=1e-15, epsrel=1e-13)[0]
        m1 = integrate.quad(lambda z: z * phi(z), a, b, epsabs=1e-15, epsrel=1e-13)[0]
        assert c[k] == pytest.approx(m1 / m0, abs=1e-10), k
    for k in range(levels - 1):
        assert t[k] == pytest.approx(0.5 * (c[k] + c[k + 1]), abs=1e-15)


@pytest.mark.parametrize("levels", [4, 32])
def test_mse_by_quadrature(levels):
    r = O.lloyd_max_gaussian(levels)
    c, t = r["centroids"], r["thresholds"]
    edges = [-np.inf] + list(t) + [np.inf]
    d = sum(integrate.quad(lambda z, ck=c[k]: (z - ck) ** 2 * phi(z), edges[k], edges[k + 1],
                           epsabs=1e-15, epsrel=1e-12)[0] for k in range(levels))
    assert r["mse"] == pytest.approx(d, rel=1e-9)


def test_mse_monte_carlo_32():
    c32, _, _ = O.codebook_fp32(32)
    z = np.random.default_rng(123).standard_normal(1_000_000)
    err = (z - c32.astype(np.float64)[O.nearest_centroid(z, c32)]) ** 2
    d = O.lloyd_max_gaussian(32)["mse"]
    se = err.std() / math.sqrt(err.size)
    assert abs(err.mean() - d) < 4 * se


def test_mse_ordering_and_high_rate():
    d = [O.lloyd_max_gaussian(L)["mse"] for L in (2, 4, 8, 16, 32)]
    assert all(a > b for a, b in zip(d, d[1:]))
    pd32 = math.sqrt(3) * math.pi / 2 / 32 ** 2
    assert d[-1] < pd32 and d[-1] > 0.9 * pd32


def test_fp32_codebook_symmetry_and_order():
    c32, mid64, b32 = O.codebook_fp32(32)
    assert c32.dtype == np.float32 and c32.shape == (32,)
    assert np.all(c32[::-1] == -c32)                    # bit-exact symmetry
    assert np.all(np.diff(c32) > 0)
    assert mid64[15] == 0.0 and b32[15] == 0.0
    assert np.all(mid64 == (c32[:-1].astype(np.float64) + c32[1:]) / 2)


def test_fp32_rounding_is_unambiguous():
    """Every fp64 centroid lies far (>1e-12 relative) from an fp32 rounding
    midpoint, so any converged solver rounds it to the same fp32 value."""
    c64 = O.lloyd_max_gaussian(32)["centroids"]
    for v in c64:
        f = np.float32(v)
        up = np.nextafter(f, np.float32(np.inf))
        dn = np.nextafter(f, np.float32(-np.inf))
        for nb in (up, dn):
            midpoint = (float(f) + float(nb)) / 2
            assert abs(v - midpoint) > 1e-12 * abs(v)
