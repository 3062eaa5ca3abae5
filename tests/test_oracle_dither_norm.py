"""Pins of the oracle's dithered quantization and corrected norm.

Dithered HD ("Minimum Distortion Quantization with Specified Output Distribution" page,
third abstract): HD, then a random scalar offset subtracted before quantizing; the page
claims the result is unbiased with MSE (pi sqrt(3)/2 + o(1)) 4^-b.  Corrected norm
("tq-kv" crate documentation: the single-key compress returns a corrected norm).

The expectations over the offset are taken here by exact piecewise integration: between
two consecutive points where y - xi crosses a boundary the index is constant, so the
reconstruction is linear in xi (its mean over a piece is its value at the piece's middle)
and the squared error is quadratic (Simpson's rule on the piece is exact)."""
import math

import numpy as np
import pytest
from scipy import integrate

from oracle import codebook as cb
from oracle import layout as lay
from oracle import quant as qt
from oracle import rotation as rot
from workloads import hadamard_signs

D = 128


def _grid(bits, step):
    n = 2 ** bits
    c = (np.arange(n) - (n - 1) / 2.0) * step
    return c, 0.5 * (c[:-1] + c[1:])


def _expect_over_offset(y, c, beta, step):
    """(E[y_hat], E[(y_hat - y)^2]) over xi ~ U[-step/2, step/2) of the oracle's
    y_hat = c[Quant(y - xi)] + xi, integrated exactly piece by piece."""
    lo, hi = -step / 2.0, step / 2.0
    cuts = np.sort(np.concatenate([[lo, hi], [y - b for b in beta if lo < y - b < hi]]))
    mean = sq = 0.0
    for a, b in zip(cuts[:-1], cuts[1:]):
        if b <= a:
            continue
        mid = 0.5 * (a + b)
        idx = qt.quantize(np.array([[y - mid]]), beta)
        yh = lambda xi: float(qt.dequantize_dithered(idx, c, np.array([xi]))[0, 0])
        w = (b - a) / step
        mean += w * yh(mid)
        sq += w * ((yh(a) - y) ** 2 + 4 * (yh(mid) - y) ** 2 + (yh(b) - y) ** 2) / 6.0
    return mean, sq


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_offset_makes_reconstruction_unbiased_with_uniform_error(bits):
    step = cb.dither_step(bits, D)
    c, beta = _grid(bits, step)
    A = c[-1]
    rng = np.random.default_rng(bits)
    for y in np.concatenate([rng.uniform(-A, A, 40), [0.0, A, -A, beta[0], beta[-1]]]):
        m, e2 = _expect_over_offset(float(y), c, beta, step)
        assert abs(m - y) < 1e-14
        assert abs(e2 - step * step / 12.0) < 1e-15
    # beyond the outer levels every offset picks the outer level: bias and the extra error
    for y in (A + 0.3 * step, A + 2.5 * step, -A - 1.7 * step):
        m, e2 = _expect_over_offset(y, c, beta, step)
        assert abs(m - math.copysign(A, y)) < 1e-14
        assert abs(e2 - (step * step / 12.0 + (abs(y) - A) ** 2)) < 1e-14


@pytest.mark.parametrize("density", ["beta", "gauss"])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_dither_mse_closed_form_against_quadrature(bits, density):
    # D(delta) from the tail moments equals the per-coordinate error above integrated
    # against f_X by adaptive quadrature, at the optimum and away from it
    pdf = cb.DENSITIES[density][0]
    step0 = cb.dither_step(bits, D, density)
    for step in (0.6 * step0, step0, 1.7 * step0):
        A = (2 ** bits - 1) * step / 2.0
        end = 1.0 if density == "beta" else 40.0 / math.sqrt(D)
        tail, _ = integrate.quad(lambda t: (t - A) ** 2 * float(pdf(t, D)), A, end, epsabs=1e-16,
                                 epsrel=1e-12, limit=200) if A < end else (0.0, 0.0)
        ref = step * step / 12.0 + 2.0 * tail
        assert abs(cb.dither_mse(step, bits, D, density) - ref) <= 1e-10 * ref


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_dither_step_minimises_the_mse(bits):
    s = cb.dither_step(bits, D)
    f = lambda x: cb.dither_mse(x, bits, D)
    for eps in (1e-3, 1e-2, 1e-1):
        assert f(s * (1 + eps)) > f(s) and f(s * (1 - eps)) > f(s)
    # the Beta density tends to N(0, 1/d): the steps agree in units of 1/sqrt(d) for large d
    big = 1 << 20
    assert abs(cb.dither_step(bits, big) * math.sqrt(big) - cb.dither_step(bits, big, "gauss") * math.sqrt(big)) < 1e-4


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_dither_codebook_is_a_symmetric_uniform_grid(bits):
    c, b = cb.dither_codebook_f32(bits, D)
    assert c.dtype == np.float32 and b.dtype == np.float32 and len(c) == 2 ** bits and len(b) == 2 ** bits - 1
    step = cb.dither_step(bits, D)
    np.testing.assert_allclose(np.diff(c.astype(np.float64)), step, rtol=1e-6)
    np.testing.assert_array_equal(c, -c[::-1])
    np.testing.assert_allclose(b.astype(np.float64), 0.5 * (c[:-1].astype(np.float64) + c[1:]), rtol=1e-6)
    assert b[len(b) // 2] == 0.0


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_mse_claim_on_the_mean(bits):
    # the page: MSE (pi sqrt(3)/2 + o(1)) 4^-b for a unit vector, o(1) vanishing as the levels
    # grow.  The uniform-grid reading meets the constant itself for b <= 3 and lies within
    # 7 % of it at b = 4 (d = 128), where the o(1) term is not yet small.
    claim = math.pi * math.sqrt(3.0) / 2.0 * 4.0 ** -bits
    mse = D * cb.dither_mse(cb.dither_step(bits, D), bits, D)
    assert mse <= claim * (1.0 if bits <= 3 else 1.07)


@pytest.mark.parametrize("bits", [2, 3])
def test_dithered_compress_end_to_end(bits):
    # the whole oracle path (norm, HD, offset, fp16 storage, un-rotation): over many offsets
    # the reconstruction of one vector averages to the vector (all its coordinates lie inside
    # the grid) and its squared error to n^2 d delta^2 / 12; reconstructing without adding the
    # offset back (error 2x) or subtracting it with the wrong sign (5x) fails the second check
    rng = np.random.default_rng(10 + bits)
    R = rot.hd_matrix(hadamard_signs(D, 3))
    c, b = cb.dither_codebook_f32(bits, D)
    step = float(c[1]) - float(c[0])
    A = float(c[-1])
    # a vector whose rotated coordinates all lie inside the grid: |y_i| close to 1/sqrt(d)
    y = rng.choice([-1.0, 1.0], D) * rng.uniform(0.8, 1.2, D)
    y /= np.linalg.norm(y)
    assert np.max(np.abs(y)) < A
    x = 2.0 * rot.unrotate(R, y[None])[0]
    n_draw = 6000
    X = np.repeat(x[None], n_draw, axis=0)
    xi = rng.uniform(-step / 2, step / 2, n_draw)
    comp = qt.compress_mse(X, R, c, b, offsets=xi)
    np.testing.assert_array_equal(comp.offset, qt.fp16_offset(xi))
    xh = qt.reconstruct_mse(comp.idx, comp.norm, R, c, comp.offset)
    n = np.linalg.norm(x)
    se = np.linalg.norm(xh - x[None], axis=1) ** 2
    target = n * n * D * step * step / 12.0
    assert abs(se.mean() - target) < 0.1 * target
    bias = np.abs(xh.mean(axis=0) - x).max()
    assert bias < 5 * n * step / math.sqrt(12.0 * n_draw) + 1e-3 * n


def test_zero_offset_is_plain_quantization():
    c, b = cb.dither_codebook_f32(3, D)
    R = rot.hd_matrix(hadamard_signs(D, 1))
    X = np.random.default_rng(4).standard_normal((20, D))
    plain = qt.compress_mse(X, R, c, b)
    dith = qt.compress_mse(X, R, c, b, offsets=np.zeros(20))
    np.testing.assert_array_equal(plain.idx, dith.idx)
    np.testing.assert_array_equal(plain.norm, dith.norm)
    np.testing.assert_allclose(qt.reconstruct_mse(plain.idx, plain.norm, R, c),
                               qt.reconstruct_mse(dith.idx, dith.norm, R, c, dith.offset), atol=0)


def test_offset_regions_hand_placed():
    # KD and VD come after every other region; the offsets are fp16, little endian:
    # 0.5 = 0x3800, -0.25 = 0xB400, 0.125 = 0x3000, -2 = 0xC000
    fmt = lay.Format(key_bits=2, key_qjl=False, value_bits=2, dither=True)
    plain = lay.Format(key_bits=2, key_qjl=False, value_bits=2)
    reg = fmt.regions()
    P = fmt.page_tokens
    assert reg["KD"] == (plain.block_bytes, 2 * P) and reg["VD"] == (plain.block_bytes + 2 * P, 2 * P)
    assert fmt.block_bytes == plain.block_bytes + 4 * P
    k = qt.Compressed(idx=np.zeros((2, D), dtype=np.int64), norm=np.ones(2), y=None,
                      offset=np.array([0.5, -0.25]))
    v = qt.Compressed(idx=np.zeros((2, D), dtype=np.int64), norm=np.ones(2), y=None,
                      offset=np.array([0.125, -2.0]))
    cache = lay.empty_cache(fmt, 1, 1)
    lay.write_sequence(cache, fmt, 0, 0, [0], k, v)
    blk = cache[0, 0, 0]
    kd, vd = reg["KD"][0], reg["VD"][0]
    assert list(blk[kd:kd + 4]) == [0x00, 0x38, 0x00, 0xB4]
    assert list(blk[vd:vd + 4]) == [0x00, 0x30, 0x00, 0xC0]
    u = lay.read_sequence(cache, fmt, 0, 0, [0], 2)
    np.testing.assert_array_equal(u.k_offset, [0.5, -0.25])
    np.testing.assert_array_equal(u.v_offset, [0.125, -2.0])


# ---------------------------------------------------------------------------
# corrected norm
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("dither", [False, True])
def test_corrected_norm_reconstruction_keeps_the_norm(bits, dither):
    rng = np.random.default_rng(bits)
    R = rot.hd_matrix(hadamard_signs(D, 2))
    c, b = cb.dither_codebook_f32(bits, D) if dither else cb.codebook_f32(bits, D)
    X = rng.standard_normal((30, D)) * rng.uniform(0.1, 10.0, (30, 1))
    off = rng.uniform(-0.5, 0.5, 30) * (float(c[1]) - float(c[0])) if dither else None
    plain = qt.compress_mse(X, R, c, b, offsets=off)
    corr = qt.compress_mse(X, R, c, b, offsets=off, corrected_norm=True)
    np.testing.assert_array_equal(plain.idx, corr.idx)
    xp = qt.reconstruct_mse(plain.idx, plain.norm, R, c, plain.offset)
    xc = qt.reconstruct_mse(corr.idx, corr.norm, R, c, corr.offset)
    # same direction, and the input's norm up to the fp16 rounding of the stored value
    cos = np.sum(xp * xc, axis=1) / (np.linalg.norm(xp, axis=1) * np.linalg.norm(xc, axis=1))
    np.testing.assert_allclose(cos, 1.0, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(xc, axis=1), np.linalg.norm(X, axis=1), rtol=2.0 ** -11)
    # the plain MSE reconstruction is shorter than the input (each cell's centroid is its mean)
    if not dither:
        assert np.mean(np.linalg.norm(xp, axis=1) / np.linalg.norm(X, axis=1)) < 1.0


def test_corrected_norm_one_bit_closed_form():
    # b = 1: every coordinate reconstructs to +-c_1, so ||y_hat|| = sqrt(d) c_1
    R = rot.hd_matrix(hadamard_signs(D, 6))
    c, b = cb.codebook_f32(1, D)
    X = np.random.default_rng(8).standard_normal((10, D))
    corr = qt.compress_mse(X, R, c, b, corrected_norm=True)
    ref = qt.fp16_round(np.linalg.norm(X, axis=1) / (math.sqrt(D) * float(c[1])))
    np.testing.assert_array_equal(corr.norm, ref)


def test_corrected_norm_of_zero_vector_is_zero():
    R = rot.hd_matrix(hadamard_signs(D, 6))
    c, b = cb.codebook_f32(2, D)
    corr = qt.compress_mse(np.zeros((2, D)), R, c, b, corrected_norm=True)
    np.testing.assert_array_equal(corr.norm, [0.0, 0.0])
