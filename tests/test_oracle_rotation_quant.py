"""Pins of the oracle's rotation, quantization and packing."""
import math

import numpy as np
import pytest
from scipy import linalg

from oracle import codebook as cb
from oracle import layout as lay
from oracle import quant as qt
from oracle import rotation as rot
from workloads import hadamard_signs, haar_matrix


@pytest.mark.parametrize("d", [2, 4, 8, 64, 128, 256])
def test_sylvester_matches_library_and_recursion(d):
    H = rot.sylvester_hadamard(d)
    np.testing.assert_array_equal(H, linalg.hadamard(d) / math.sqrt(d))
    # the page's recursive definition: H_2 = [[1,1],[1,-1]]/sqrt2, H_2n = H_2 (x) H_n
    h = np.array([[1.0]])
    h2 = np.array([[1.0, 1.0], [1.0, -1.0]]) / math.sqrt(2)
    while h.shape[0] < d:
        h = np.kron(h2, h)
    np.testing.assert_allclose(H, h, atol=1e-15)


def test_hd_spreads_energy_page_value(golden):
    g = golden["hd_spread_max_abs"]
    d = g["d"]
    R = rot.hd_matrix(hadamard_signs(d, 0))
    e0 = np.zeros(d)
    e0[0] = 1.0
    y = rot.rotate(R, e0[None])[0]
    assert abs(np.max(np.abs(y)) - g["value"]) < g["tol"]
    np.testing.assert_allclose(np.abs(y), 1 / math.sqrt(d), rtol=1e-14)


@pytest.mark.parametrize("kind", ["hd", "haar"])
def test_rotation_orthogonal_and_norm_preserving(kind):
    d = 128
    R = rot.hd_matrix(hadamard_signs(d, 5)) if kind == "hd" else haar_matrix(d, 5)
    tol = 1e-14 if kind == "hd" else 1e-6  # the Haar matrix is fp32-rounded
    np.testing.assert_allclose(R.T @ R, np.eye(d), atol=tol)
    x = np.random.default_rng(0).standard_normal((50, d))
    np.testing.assert_allclose(np.linalg.norm(rot.rotate(R, x), axis=1),
                               np.linalg.norm(x, axis=1), rtol=10 * tol)
    np.testing.assert_allclose(rot.unrotate(R, rot.rotate(R, x)), x, atol=1e-12 if kind == "hd" else 1e-5)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_centroid_maps_to_itself(bits):
    # "Quantize -> dequantize should map each centroid exactly to itself"
    c, b = cb.codebook_f32(bits, 128)
    idx = qt.quantize(c.astype(np.float64), b)
    np.testing.assert_array_equal(idx, np.arange(2 ** bits))
    np.testing.assert_array_equal(qt.dequantize(idx, c), c.astype(np.float64))


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_value_near_centroid_gets_its_index(bits):
    c, b = cb.codebook_f32(bits, 128)
    gap = np.min(np.diff(c.astype(np.float64)))
    rng = np.random.default_rng(bits)
    for i, ci in enumerate(c.astype(np.float64)):
        v = ci + rng.uniform(-0.4, 0.4, 100) * gap
        assert np.all(qt.quantize(v, b) == i)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_bucketize_equals_nearest_centroid_brute_force(bits):
    c, b = cb.codebook_f32(bits, 128)
    y = np.random.default_rng(7).normal(0, 1 / math.sqrt(128), 200000)
    idx = qt.quantize(y, b)
    dist = np.abs(y[:, None] - c.astype(np.float64)[None, :])
    brute = np.argmin(dist, axis=1)
    # they may differ only where two centroids are equidistant up to fp32 boundary rounding
    diff = idx != brute
    if np.any(diff):
        sd = np.sort(dist[diff], axis=1)
        assert np.all(sd[:, 1] - sd[:, 0] < 1e-7)


def test_tie_goes_to_lower_index():
    c, b = cb.codebook_f32(3, 128)
    bb = b.astype(np.float64)
    np.testing.assert_array_equal(qt.quantize(bb, b), np.arange(7))
    assert qt.quantize(np.array([-0.0]), b)[0] == 3


def test_norm_storage_and_overflow():
    x = np.array([[3.0, 4.0] + [0.0] * 126])
    R = rot.hd_matrix(hadamard_signs(128, 0))
    c, b = cb.codebook_f32(2, 128)
    comp = qt.compress_mse(x, R, c, b)
    assert comp.norm[0] == 5.0
    with pytest.raises(qt.NormOverflow):
        qt.compress_mse(np.full((1, 128), 7000.0), R, c, b)
    z = qt.compress_mse(np.zeros((1, 128)), R, c, b)
    assert z.norm[0] == 0.0
    np.testing.assert_array_equal(qt.reconstruct_mse(z.idx, z.norm, R, c), 0.0)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_unit_vector_mse_within_bounds(golden, bits):
    # "MSE distortion per vector <= sqrt(3) pi/2 4^-b": tested on the mean over 4096 unit
    # vectors (the theory bounds the expectation), and >= the lower bound 4^-b
    d = 128
    rng = np.random.default_rng(100 + bits)
    x = rng.standard_normal((4096, d))
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    R = rot.hd_matrix(hadamard_signs(d, bits))
    c, b = cb.codebook_f32(bits, d)
    comp = qt.compress_mse(x, R, c, b)
    xh = qt.reconstruct_mse(comp.idx, comp.norm, R, c)
    mse = np.sum((x - xh) ** 2, axis=1)
    assert mse.mean() <= math.sqrt(3) * math.pi / 2 * 4.0 ** -bits
    assert mse.mean() >= 4.0 ** -bits


def test_more_bits_lower_reconstruction_error_and_norm_cosine():
    d = 128
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2048, d)) * np.exp(rng.normal(0, 0.5, d))
    R = rot.hd_matrix(hadamard_signs(d, 0))
    prev = np.inf
    for bits in (1, 2, 3, 4):
        c, b = cb.codebook_f32(bits, d)
        comp = qt.compress_mse(x, R, c, b)
        xh = qt.reconstruct_mse(comp.idx, comp.norm, R, c)
        err = np.mean(np.sum((x - xh) ** 2, axis=1) / np.sum(x ** 2, axis=1))
        assert err < prev
        prev = err
        # stored norm is the fp16 rounding of ||x||
        np.testing.assert_allclose(comp.norm, np.linalg.norm(x, axis=1), rtol=2 ** -11)
        cos = np.sum(x * xh, axis=1) / np.linalg.norm(x, axis=1) / np.linalg.norm(xh, axis=1)
        assert cos.mean() > {1: 0.75, 2: 0.92, 3: 0.98, 4: 0.994}[bits]
        # reconstruction norm approximately preserved
        ratio = np.linalg.norm(xh, axis=1) / np.linalg.norm(x, axis=1)
        assert abs(ratio.mean() - 1) < {1: 0.25, 2: 0.1, 3: 0.03, 4: 0.01}[bits]


@pytest.mark.parametrize("name", ["b1_idx_j_mod_2", "b2_idx_j_mod_4", "b3_idx_j_mod_8",
                                  "b4_idx_j_mod_16"])
def test_packing_matches_hand_derived_bytes(packing_golden, name):
    g = packing_golden[name]
    bits = g["bits"]
    idx = (np.arange(128) % (2 ** bits))[None, :]
    got = lay.bits_to_bytes(lay.code_bits(idx, bits))[0]
    assert got.tobytes().hex() == g["bytes_hex"]
    back = lay.index_from_bits(lay.bytes_to_bits(got[None]), bits, 128)
    np.testing.assert_array_equal(back, idx)


def test_merged_key_packing_matches_hand_derived_bytes(packing_golden):
    g = packing_golden["k3_qjl_merged_idx_j_mod_8_sigma_j_mod_2"]
    j = np.arange(128)
    idx, sigma = (j % 8)[None, :], (j % 2)[None, :]
    got = lay.bits_to_bytes(lay.merged_key_bits(idx, sigma))[0]
    assert got.tobytes().hex() == g["bytes_hex"]
    bidx, bsig = lay.merged_key_from_bits(lay.bytes_to_bits(got[None]), 128)
    np.testing.assert_array_equal(bidx, idx)
    np.testing.assert_array_equal(bsig, sigma.astype(bool))


def test_sign_plane_permutation_is_a_bijection():
    pos = lay.sign_plane_position(np.arange(128))
    assert sorted(pos.tolist()) == list(range(128))
    assert np.all(pos // 32 == np.arange(128) // 32)


@pytest.mark.parametrize("name", ["c2_regions", "c2_value_qjl_regions"])
def test_region_offsets_match_hand_derivation(packing_golden, name):
    g = packing_golden[name]
    fmt = lay.Format(**g["format"])
    reg = fmt.regions()
    for k, v in g["offsets"].items():
        assert reg[k][0] == v
    assert fmt.block_bytes == g["total"]


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_stored_code_sign_magnitude_identity(bits):
    # c[idx] == (+1 if s else -1) * c[h + r] on the symmetric codebook
    c, _ = cb.codebook_f32(bits, 128)
    idx = np.arange(2 ** bits)
    s, r = lay.stored_code(idx, bits)
    h = 2 ** (bits - 1)
    np.testing.assert_array_equal(c[idx], np.where(s == 1, 1, -1) * c[h + r])
    np.testing.assert_array_equal(lay.index_from_code(s, r, bits), idx)


def test_page_round_trip_with_partial_last_page():
    fmt = lay.Format(key_bits=3, key_qjl=True, value_bits=2, page_tokens=256)
    n = 600
    rng = np.random.default_rng(1)
    K = qt.Compressed(idx=rng.integers(0, 8, (n, 128)), norm=rng.uniform(0, 50, n).astype(np.float16).astype(float),
                      y=None, rnorm=rng.uniform(0, 5, n).astype(np.float16).astype(float),
                      sigma=rng.integers(0, 2, (n, 128)).astype(bool))
    V = qt.Compressed(idx=rng.integers(0, 4, (n, 128)), norm=rng.uniform(0, 50, n).astype(np.float16).astype(float), y=None)
    cache = lay.empty_cache(fmt, num_pages=5, kv_heads=2)
    pages = [4, 0, 2]
    lay.write_sequence(cache, fmt, 0, 1, pages, K, V)
    u = lay.read_sequence(cache, fmt, 0, 1, pages, n)
    np.testing.assert_array_equal(u.k_idx, K.idx)
    np.testing.assert_array_equal(u.v_idx, V.idx)
    np.testing.assert_array_equal(u.k_sigma, K.sigma)
    np.testing.assert_array_equal(u.k_norm, K.norm)
    np.testing.assert_array_equal(u.k_rnorm, K.rnorm)
    np.testing.assert_array_equal(u.v_norm, V.norm)
    # token 300 = page 1 (physical 0) slot 44: its second key chunk sits at (1*256+44)*16 of KC
    o, _ = fmt.regions()["KC"]
    tok_bytes = lay.bits_to_bytes(lay.merged_key_bits(K.idx[300:301], K.sigma[300:301]))[0]
    blk = cache[0, 0, 1]
    assert blk[o + (256 + 44) * 16: o + (256 + 44) * 16 + 16].tobytes() == tok_bytes[16:32].tobytes()
    assert not cache[0, :, 0].any()


def test_value_qjl_page_round_trip_and_hand_placed_bytes():
    # values with QJL: the residual's sign bits go to VS (bit i = sigma_i, 16-byte chunk per
    # token) and its fp16 norm to VR, both after VC (offsets 30208 and 34304 for this format)
    fmt = lay.Format(key_bits=3, key_qjl=True, value_bits=3, page_tokens=256, value_qjl=True)
    n = 300
    rng = np.random.default_rng(2)
    K = qt.Compressed(idx=rng.integers(0, 8, (n, 128)), norm=rng.uniform(0, 50, n).astype(np.float16).astype(float),
                      y=None, rnorm=rng.uniform(0, 5, n).astype(np.float16).astype(float),
                      sigma=rng.integers(0, 2, (n, 128)).astype(bool))
    vs = np.zeros((n, 128), dtype=bool)
    vs[5, 0] = vs[5, 9] = vs[5, 127] = True  # token 5: bits 0, 9 and 127 of its chunk
    V = qt.Compressed(idx=rng.integers(0, 8, (n, 128)), norm=rng.uniform(0, 50, n).astype(np.float16).astype(float),
                      y=None, rnorm=np.full(n, 1.5), sigma=vs)
    cache = lay.empty_cache(fmt, num_pages=3, kv_heads=1)
    lay.write_sequence(cache, fmt, 0, 0, [2, 0], K, V)
    u = lay.read_sequence(cache, fmt, 0, 0, [2, 0], n)
    np.testing.assert_array_equal(u.v_sigma, vs)
    np.testing.assert_array_equal(u.v_rnorm, V.rnorm)
    np.testing.assert_array_equal(u.v_idx, V.idx)
    np.testing.assert_array_equal(u.k_sigma, K.sigma)
    blk = cache[0, 2, 0]
    assert blk[30208 + 5 * 16: 30208 + 6 * 16].tobytes().hex() == "0102" + "00" * 13 + "80"
    assert blk[34304 + 10: 34304 + 12].tobytes() == np.float16(1.5).tobytes()
    # token 256 is slot 0 of the second page (physical 0)
    assert cache[0, 0, 0][34304: 34306].tobytes() == np.float16(1.5).tobytes()
