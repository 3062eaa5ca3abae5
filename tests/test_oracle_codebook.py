"""Pins of the oracle's codebook against what the pages and the mathematics fix.

Each test names what it pins; none re-types the oracle's own formula.
"""
import math

import numpy as np
import pytest
from scipy import integrate, stats

from oracle import codebook as cb


@pytest.mark.parametrize("d", [8, 64, 128])
def test_beta_pdf_matches_library_beta_law(d):
    # f_X(t) dt is the law of 2B - 1, B ~ Beta((d-1)/2, (d-1)/2) (the page's KS check uses this law)
    a = (d - 1) / 2
    t = np.linspace(-0.99, 0.99, 397)
    ref = stats.beta.pdf((t + 1) / 2, a, a) / 2
    np.testing.assert_allclose(cb.beta_pdf(t, d), ref, rtol=1e-10, atol=1e-300)


@pytest.mark.parametrize("d", [4, 16, 128])
def test_beta_closed_forms_match_quadrature(d):
    # cell mass and first moment used by Lloyd-Max against adaptive quadrature of the density
    lo, hi = -0.3, 0.17
    mass, _ = integrate.quad(lambda x: float(cb.beta_pdf(x, d)), lo, hi, epsabs=1e-15, epsrel=1e-13)
    mom, _ = integrate.quad(lambda x: x * float(cb.beta_pdf(x, d)), lo, hi, epsabs=1e-15, epsrel=1e-13)
    assert abs((cb.beta_cdf(hi, d) - cb.beta_cdf(lo, d)) - mass) < 1e-12
    assert abs(cb.beta_first_moment(lo, hi, d) - mom) < 1e-12
    total, _ = integrate.quad(lambda x: float(cb.beta_pdf(x, d)), -1, 1, epsabs=1e-14)
    assert abs(total - 1.0) < 1e-10


def test_gauss_closed_forms_match_quadrature():
    d = 128
    lo, hi = -0.05, 0.11
    mass, _ = integrate.quad(lambda x: float(cb.gauss_pdf(x, d)), lo, hi, epsabs=1e-15)
    mom, _ = integrate.quad(lambda x: x * float(cb.gauss_pdf(x, d)), lo, hi, epsabs=1e-15)
    assert abs((cb.gauss_cdf(hi, d) - cb.gauss_cdf(lo, d)) - mass) < 1e-12
    assert abs(cb.gauss_first_moment(lo, hi, d) - mom) < 1e-12


def test_ks_unit_sphere_coordinates_follow_the_density(golden):
    g = golden["beta_ks_pvalue_min"]
    d = g["d"]
    rng = np.random.default_rng(11)
    X = rng.standard_normal((g["samples"], d))
    X /= np.linalg.norm(X, axis=1, keepdims=True)
    p = stats.kstest(X[:, 0], lambda t: cb.beta_cdf(t, d)).pvalue
    assert p > g["value"]


@pytest.mark.parametrize("d", [8, 64, 128])
def test_one_bit_beta_centroid_closed_form(d):
    # b = 1: centroids +-E|X| = +-Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
    c, beta, _ = cb.lloyd_max(1, d, "beta")
    ref = math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)
    np.testing.assert_allclose(c, [-ref, ref], rtol=1e-12)
    assert beta[0] == 0.0


def test_one_bit_gaussian_codebook_page_value(golden):
    d = golden["onebit_codebook"]["d"]
    c, _, _ = cb.lloyd_max(1, d, "gauss")
    ref = math.sqrt(2 / (math.pi * d))
    np.testing.assert_allclose(c, [-ref, ref], rtol=1e-12)


def test_two_bit_gaussian_codebook_page_value(golden):
    g = golden["gauss_2bit_codebook_times_sqrt_d"]
    c, _, _ = cb.lloyd_max(2, g["d"], "gauss")
    np.testing.assert_allclose(c * math.sqrt(g["d"]), g["value"], atol=g["tol"])


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_beta_codebook_close_to_gaussian_at_d128(golden, bits):
    g = golden["beta_close_to_gaussian"]
    cbeta, _, _ = cb.lloyd_max(bits, g["d"], "beta")
    cgau, _, _ = cb.lloyd_max(bits, g["d"], "gauss")
    np.testing.assert_allclose(cbeta, cgau, rtol=g["rel_tol"])


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("density", ["beta", "gauss"])
def test_lloyd_max_fixed_point_by_quadrature(bits, density):
    # boundaries are midpoints and centroids are conditional means, checked with quad
    d = 128
    c, beta, _ = cb.lloyd_max(bits, d, density)
    np.testing.assert_allclose(beta, 0.5 * (c[:-1] + c[1:]), atol=1e-15)
    pdf = cb.DENSITIES[density][0]
    s = 1 / math.sqrt(d)
    edges = np.concatenate([[-1.0 if density == "beta" else -40 * s], beta,
                            [1.0 if density == "beta" else 40 * s]])
    for i in range(len(c)):
        m0, _ = integrate.quad(lambda x: float(pdf(x, d)), edges[i], edges[i + 1],
                               epsabs=1e-15, epsrel=1e-13, limit=200)
        m1, _ = integrate.quad(lambda x: x * float(pdf(x, d)), edges[i], edges[i + 1],
                               epsabs=1e-16, epsrel=1e-13, limit=200)
        assert abs(m1 / m0 - c[i]) < 1e-10
    assert np.all(np.diff(c) > 0)
    np.testing.assert_array_equal(c, -c[::-1])


def test_unit_vector_mse_page_values(golden):
    g = golden["unit_mse"]
    d = g["d"]
    for b, ref in g["value"].items():
        c, _, _ = cb.lloyd_max(int(b), d, "beta")
        assert abs(d * cb.distortion(c, d, "beta") - ref) < g["tol"]


def test_gaussian_one_bit_mse_closed_form():
    # one bit, Gaussian law: total MSE d * C = 1 - 2/pi
    d = 128
    c, _, _ = cb.lloyd_max(1, d, "gauss")
    assert abs(d * cb.distortion(c, d, "gauss") - (1 - 2 / math.pi)) < 1e-9


def test_mse_bounds_and_monotonicity(golden):
    d = 128
    vals = []
    for b in range(1, 5):
        c, _, _ = cb.lloyd_max(b, d, "beta")
        mse = d * cb.distortion(c, d, "beta")
        vals.append(mse)
        assert mse <= math.sqrt(3) * math.pi / 2 * 4.0 ** -b
        assert mse >= 4.0 ** -b
    assert all(vals[i + 1] < vals[i] for i in range(3))
    g = golden["bound_ratio"]
    assert abs(math.sqrt(3) * math.pi / 2 - g["value"]) < g["tol"]
    assert abs(vals[0] / 0.25 - g["b1_gap"]) < g["b1_tol"]


def _exact_mse_grid(codebooks, d, n=40001):
    # MSE of nearest-centroid quantization, by trapezoid on a fine grid (brute force)
    t = np.linspace(-1, 1, n)
    w = cb.beta_pdf(t, d)
    out = []
    for c in codebooks:
        err = np.min((t[:, None] - np.asarray(c)[None, :]) ** 2, axis=1)
        out.append(np.trapezoid(err * w, t))
    return np.array(out)


@pytest.mark.parametrize("d", [4, 8])
def test_brute_force_one_bit_tiny_d(d):
    c, _, _ = cb.lloyd_max(1, d, "beta")
    grid = np.linspace(0.05, 0.95, 901)
    mse = _exact_mse_grid([[-a, a] for a in grid], d)
    a0 = grid[np.argmin(mse)]
    fine = np.linspace(a0 - 0.002, a0 + 0.002, 401)
    mse = _exact_mse_grid([[-a, a] for a in fine], d)
    assert abs(fine[np.argmin(mse)] - c[1]) < 2e-4


@pytest.mark.parametrize("d", [4, 8])
def test_brute_force_two_bit_tiny_d(d):
    c, _, _ = cb.lloyd_max(2, d, "beta")
    lo1, hi1, lo2, hi2 = 0.01, 0.8, 0.05, 0.99
    best = None
    for _ in range(4):
        a1s = np.linspace(lo1, hi1, 25)
        a2s = np.linspace(lo2, hi2, 25)
        books = [[-a2, -a1, a1, a2] for a1 in a1s for a2 in a2s if a2 > a1]
        mse = _exact_mse_grid(books, d, n=8001)
        best = books[int(np.argmin(mse))]
        s1, s2 = (hi1 - lo1) / 24 * 2, (hi2 - lo2) / 24 * 2
        lo1, hi1 = best[2] - s1, best[2] + s1
        lo2, hi2 = best[3] - s2, best[3] + s2
    assert abs(best[2] - c[2]) < 2e-3
    assert abs(best[3] - c[3]) < 2e-3


def test_codebook_f32_is_rounding_of_double():
    c, b, _ = cb.lloyd_max(3, 128, "beta")
    c32, b32 = cb.codebook_f32(3, 128, "beta")
    assert c32.dtype == np.float32 and b32.dtype == np.float32
    np.testing.assert_array_equal(c32, c.astype(np.float32))
    np.testing.assert_array_equal(b32, b.astype(np.float32))
    assert b32[3] == 0.0
