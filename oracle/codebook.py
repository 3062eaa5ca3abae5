"""Lloyd-Max codebooks on the rotated-coordinate density (oracle; test infrastructure).

Source: "TurboQuant explained" (Mobilint blog)
  * section "Coordinates Become Predictable After Rotation": a coordinate of a
    randomly rotated unit vector in R^d has density
        f_X(t) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) * (1 - t^2)^((d-3)/2),  t in [-1, 1],
    which tends to N(0, 1/d); equivalently (t+1)/2 ~ Beta((d-1)/2, (d-1)/2)
    (the page's sanity check uses exactly this Beta law).
  * section "Designing the Optimal Codebook Without Data": the optimal b-bit
    scalar quantizer minimises C(f_X, b) = sum_i int |x - c_i|^2 f_X(x) dx and is
    found by Lloyd-Max: (1) boundaries are the midpoints of adjacent centroids,
    (2) each centroid is the conditional mean E[X | X in its cell], (3) repeat
    until convergence.  The sample-based variant printed there starts from
    linspace(-2 sigma, 2 sigma, 2^b); the same start is used here with
    sigma = 1/sqrt(d).
  * "turboquant_cutile" function list: the codebook is returned as sorted
    float32 tensors, centroids (2^b,) and boundaries (2^b - 1,).
  * "tq-kv" crate documentation, module codebook: a Gaussian-fitted variant.

Dithered quantization ("Minimum Distortion Quantization with Specified Output
Distribution" page, third abstract: one randomized Hadamard transform, then a random
scalar offset subtracted before a scalar quantizer; unbiased, MSE near
(pi sqrt(3)/2) 4^-b):
  * reading: the scalar quantizer is a uniform grid of n = 2^b levels with step
    delta, c_j = (j - (n-1)/2) delta, boundaries at the midpoints, and the offset xi
    is uniform on [-delta/2, delta/2), one per vector; a coordinate y is coded as
    idx = Quant(y - xi) and reconstructed as c[idx] + xi (subtractive dither, which
    is what makes the reconstruction unbiased inside the grid's range);
  * for a coordinate y the expected squared error over xi is exactly
        delta^2/12 + max(|y| - A, 0)^2,   A = (n-1) delta / 2
    (inside the outer levels the error is uniform on one cell; beyond them the
    outer level is taken for every xi), so the per-coordinate MSE on f_X is
        D(delta) = delta^2/12 + 2 [P2(A) - 2 A P1(A) + A^2 P0(A)],
    P_k(A) = int_A^inf t^k f_X(t) dt;
  * reading: delta is the minimiser of D; dD/d delta = delta/6 - 2(n-1)[P1(A) - A P0(A)]
    is increasing in delta, so the minimiser is its unique root (found by bisection).

Readings taken where the pages are open:
  * the integrals are computed with closed forms: the cell mass is a difference
    of the regularized incomplete Beta function, and the first moment of
    f_X has the antiderivative -K (1 - t^2)^((d-1)/2) / (d - 1);
  * convergence is max |c_new - c| < 1e-13 (at most 100000 iterations);
  * the result is symmetrised, c_i = -c_{n-1-i}, which the density's symmetry
    makes exact; the middle boundary is then exactly 0;
  * the fp32 boundaries are the fp32 rounding of the double midpoints of the
    double centroids.
"""
from __future__ import annotations

import math

import numpy as np
from scipy import special


# ---------------------------------------------------------------------------
# densities
# ---------------------------------------------------------------------------

def beta_constant(d: int) -> float:
    """K = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2))."""
    return math.exp(math.lgamma(d / 2.0) - math.lgamma((d - 1) / 2.0)) / math.sqrt(math.pi)


def beta_pdf(t, d: int):
    t = np.asarray(t, dtype=np.float64)
    out = beta_constant(d) * np.power(np.clip(1.0 - t * t, 0.0, None), (d - 3) / 2.0)
    return np.where(np.abs(t) <= 1.0, out, 0.0)


def beta_cdf(t, d: int):
    """P[X <= t] for the rotated-coordinate density: (t+1)/2 ~ Beta(a, a), a = (d-1)/2."""
    a = (d - 1) / 2.0
    t = np.clip(np.asarray(t, dtype=np.float64), -1.0, 1.0)
    return special.betainc(a, a, (t + 1.0) / 2.0)


def beta_first_moment(lo, hi, d: int):
    """int_lo^hi t f_X(t) dt = K / (d-1) * [(1-lo^2)^((d-1)/2) - (1-hi^2)^((d-1)/2)]."""
    lo = np.clip(np.asarray(lo, dtype=np.float64), -1.0, 1.0)
    hi = np.clip(np.asarray(hi, dtype=np.float64), -1.0, 1.0)
    p = (d - 1) / 2.0
    return beta_constant(d) / (d - 1) * (np.power(1.0 - lo * lo, p) - np.power(1.0 - hi * hi, p))


def gauss_pdf(t, d: int):
    s = 1.0 / math.sqrt(d)
    t = np.asarray(t, dtype=np.float64)
    return np.exp(-0.5 * (t / s) ** 2) / (s * math.sqrt(2.0 * math.pi))


def gauss_cdf(t, d: int):
    return special.ndtr(np.asarray(t, dtype=np.float64) * math.sqrt(d))


def gauss_first_moment(lo, hi, d: int):
    """int_lo^hi t N(t; 0, 1/d) dt = sigma * (phi(lo/sigma) - phi(hi/sigma))."""
    s = 1.0 / math.sqrt(d)
    phi = lambda z: np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)
    lo = np.asarray(lo, dtype=np.float64)
    hi = np.asarray(hi, dtype=np.float64)
    return s * (phi(lo / s) - phi(hi / s))


DENSITIES = {
    "beta": (beta_pdf, beta_cdf, beta_first_moment, (-1.0, 1.0)),
    "gauss": (gauss_pdf, gauss_cdf, gauss_first_moment, (-np.inf, np.inf)),
}


# ---------------------------------------------------------------------------
# Lloyd-Max
# ---------------------------------------------------------------------------

def lloyd_max(bits: int, d: int, density: str = "beta", tol: float = 1e-13,
              max_iter: int = 100000) -> tuple[np.ndarray, np.ndarray, int]:
    """Lloyd-Max codebook on f_X.  Returns (centroids, boundaries, iterations), float64."""
    if bits < 1:
        raise ValueError("bits must be >= 1")
    _, cdf, m1, (lo_end, hi_end) = DENSITIES[density]
    n = 2 ** bits
    sigma = 1.0 / math.sqrt(d)
    c = np.linspace(-2.0 * sigma, 2.0 * sigma, n)
    it = 0
    for it in range(1, max_iter + 1):
        # step 1: boundaries are the midpoints of adjacent centroids
        beta = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate([[lo_end], beta, [hi_end]])
        # step 2: each centroid is the conditional mean of its cell
        mass = cdf(edges[1:], d) - cdf(edges[:-1], d)
        mom = m1(edges[:-1], edges[1:], d)
        c_new = mom / mass
        delta = np.max(np.abs(c_new - c))
        c = c_new
        # step 3: repeat until convergence
        if delta < tol:
            break
    c = 0.5 * (c - c[::-1])
    beta = 0.5 * (c[:-1] + c[1:])
    beta[n // 2 - 1] = 0.0
    return c, beta, it


def codebook_f32(bits: int, d: int, density: str = "beta") -> tuple[np.ndarray, np.ndarray]:
    """(centroids, boundaries) as sorted float32 arrays, as the function list states."""
    c, b, _ = lloyd_max(bits, d, density)
    return c.astype(np.float32), b.astype(np.float32)


def distortion(centroids, d: int, density: str = "beta") -> float:
    """C(f_X, b): expected squared error of one coordinate under nearest-centroid
    quantization, by adaptive quadrature over each Voronoi cell (scipy.integrate.quad)."""
    from scipy import integrate
    pdf, _, _, (lo_end, hi_end) = DENSITIES[density]
    c = np.asarray(centroids, dtype=np.float64)
    beta = 0.5 * (c[:-1] + c[1:])
    edges = np.concatenate([[lo_end], beta, [hi_end]])
    total = 0.0
    for i in range(len(c)):
        a, b = edges[i], edges[i + 1]
        if density == "gauss":
            s = 1.0 / math.sqrt(d)
            a = max(a, -40 * s)
            b = min(b, 40 * s)
        val, _ = integrate.quad(lambda x: (x - c[i]) ** 2 * float(pdf(x, d)), a, b,
                                epsabs=1e-15, epsrel=1e-12, limit=200)
        total += val
    return total


# ---------------------------------------------------------------------------
# dithered quantization: uniform grid, MSE-optimal step
# ---------------------------------------------------------------------------

def tail_moments(A: float, d: int, density: str = "beta") -> tuple[float, float, float]:
    """(P0, P1, P2): int_A^inf t^k f_X(t) dt for k = 0, 1, 2 and A >= 0.

    beta:  P0 = 1 - F(A); P1 from the first-moment antiderivative; with u = t^2,
           P2 = (1 / (2d)) (1 - I_{A^2}(3/2, (d-1)/2))  (B(3/2, a) / B(1/2, a) = 1/d, a = (d-1)/2).
    gauss: with s = 1/sqrt(d), z = A/s: P0 = Q(z), P1 = s phi(z), P2 = s^2 (z phi(z) + Q(z))."""
    if A < 0:
        raise ValueError("A must be >= 0")
    if density == "beta":
        if A >= 1.0:
            return 0.0, 0.0, 0.0
        P0 = float(1.0 - beta_cdf(A, d))
        P1 = float(beta_first_moment(A, 1.0, d))
        P2 = float((1.0 - special.betainc(1.5, (d - 1) / 2.0, A * A)) / (2.0 * d))
        return P0, P1, P2
    s = 1.0 / math.sqrt(d)
    z = A / s
    phi = math.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)
    Q = float(special.ndtr(-z))
    return Q, s * phi, s * s * (z * phi + Q)


def dither_mse(step: float, bits: int, d: int, density: str = "beta") -> float:
    """D(delta): expected squared error of one coordinate under the dithered uniform grid."""
    n = 2 ** bits
    A = (n - 1) * step / 2.0
    P0, P1, P2 = tail_moments(A, d, density)
    return step * step / 12.0 + 2.0 * (P2 - 2.0 * A * P1 + A * A * P0)


def dither_step(bits: int, d: int, density: str = "beta") -> float:
    """The minimiser of D: root of delta/6 - 2(n-1)[P1(A) - A P0(A)] by bisection."""
    if bits < 1:
        raise ValueError("bits must be >= 1")
    n = 2 ** bits

    def slope(step):
        A = (n - 1) * step / 2.0
        P0, P1, _ = tail_moments(A, d, density)
        return step / 6.0 - 2.0 * (n - 1) * (P1 - A * P0)

    lo = 0.0
    hi = 2.0 / (n - 1) if density == "beta" else 2.0 * 40.0 / math.sqrt(d) / (n - 1)
    while slope(hi) <= 0.0:
        hi *= 2.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if mid == lo or mid == hi:
            break
        if slope(mid) > 0.0:
            hi = mid
        else:
            lo = mid
    return 0.5 * (lo + hi)


def dither_codebook_f32(bits: int, d: int, density: str = "beta") -> tuple[np.ndarray, np.ndarray]:
    """(centroids, boundaries) of the dithered quantizer as sorted float32 arrays:
    c_j = (j - (n-1)/2) delta, boundaries (j + 1 - n/2) delta (the middle one exactly 0),
    each rounded to fp32 from double."""
    n = 2 ** bits
    step = dither_step(bits, d, density)
    j = np.arange(n, dtype=np.float64)
    c = (j - (n - 1) / 2.0) * step
    b = (np.arange(n - 1, dtype=np.float64) + 1.0 - n / 2.0) * step
    return c.astype(np.float32), b.astype(np.float32)
