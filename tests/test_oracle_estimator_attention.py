"""Pins of the oracle's QJL estimator, the two-stage quantizer and decode attention."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as att
from oracle import codebook as cb
from oracle import layout as lay
from oracle import quant as qt
from oracle import rotation as rot
from workloads import hadamard_signs, qjl_matrix, haar_matrix


def _unit(rng, n, d):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def test_qjl_estimator_unbiased_over_random_S():
    # E_S[ sqrt(pi/2)/m ||k|| <S q, sign(S k)> ] = <q, k>: mean within 4 standard errors
    rng = np.random.default_rng(21)
    d, m = 128, 128
    q = rng.standard_normal(d)
    k = 0.6 * q + rng.standard_normal(d)
    ests = []
    for _ in range(10000):
        S = rng.standard_normal((m, d))
        ests.append(att.qjl_estimate(q, k, S))
    ests = np.array(ests)
    se = ests.std(ddof=1) / math.sqrt(len(ests))
    assert abs(ests.mean() - q @ k) < 4 * se


def test_qjl_estimator_unbiased_over_many_pairs():
    # "averaging over many random pairs": mean error over pairs ~ 0 relative to its spread
    rng = np.random.default_rng(22)
    d, m = 128, 128
    S = qjl_matrix(m, d, 1)
    errs = []
    for _ in range(4000):
        q, k = rng.standard_normal(d), rng.standard_normal(d)
        errs.append(att.qjl_estimate(q, k, S) - q @ k)
    errs = np.array(errs)
    assert abs(errs.mean()) < 4 * errs.std(ddof=1) / math.sqrt(len(errs))


def test_two_stage_regression_slopes(golden):
    # MSE-only slope < 1 (biased), MSE + QJL slope ~ 1 (unbiased); page's listing, fresh Pi and S per trial
    g = golden["two_stage_slopes"]
    d = g["d"]
    rng = np.random.default_rng(23)
    c, b = cb.codebook_f32(2, d, "gauss")
    truth, mse_only, with_qjl = [], [], []
    for t in range(g["trials"]):
        x = _unit(rng, 1, d)
        y = _unit(rng, 1, d)[0]
        Pi = np.linalg.qr(rng.standard_normal((d, d)))[0]
        S = rng.standard_normal((d, d))
        comp = qt.compress_prod(x, Pi, c, b, S)
        x_mse = qt.reconstruct_mse(comp.idx, comp.norm, Pi, c)[0]
        r = x[0] - x_mse
        x_qjl = math.sqrt(math.pi / 2) / d * np.linalg.norm(r) * (S.T @ np.where(S @ r >= 0, 1.0, -1.0))
        truth.append(y @ x[0])
        mse_only.append(y @ x_mse)
        with_qjl.append(y @ (x_mse + x_qjl))
    truth = np.array(truth)
    slope = lambda e: np.dot(e, truth) / np.dot(truth, truth)
    assert slope(np.array(mse_only)) < g["mse_only_below"] - 0.05
    assert abs(slope(np.array(with_qjl)) - g["with_qjl"]) < g["with_qjl_tol"]


def test_qjl_reconstruct_is_unbiased_for_the_residual():
    # E_S[x_qjl] = r for the function the estimator uses (sign / scale / transpose pinned)
    rng = np.random.default_rng(24)
    d = 64
    r = rng.standard_normal(d) * 0.1
    acc = np.zeros(d)
    n = 20000
    for _ in range(n):
        S = rng.standard_normal((d, d))
        sigma = (S @ r >= 0)[None]
        acc += qt.qjl_reconstruct(sigma, np.array([np.linalg.norm(r)]), S)[0]
    assert np.linalg.norm(acc / n - r) < 0.05 * np.linalg.norm(r)


def test_one_bit_inner_product_bias_page_value(golden):
    g = golden["onebit_inner_product_mean"]
    d = g["d"]
    rng = np.random.default_rng(25)
    c, b = cb.codebook_f32(1, d, "gauss")
    x = _unit(rng, g["trials"], d)
    xq = qt.dequantize(qt.quantize(x, b), c)
    assert abs(np.mean(np.sum(x * xq, axis=1)) - g["value"]) < g["tol"]


@pytest.mark.parametrize("bits", [2, 3])
def test_inner_product_distortion_bounds(golden, bits):
    # D_prod of (b-1)-bit MSE + 1-bit QJL: ||y||^2/d 4^-b <= D_prod <= sqrt(3) pi^2 / d ||y||^2 4^-b
    d = 128
    rng = np.random.default_rng(26 + bits)
    c, b = cb.codebook_f32(bits - 1, d)
    n = 3000
    x = _unit(rng, n, d)
    y = rng.standard_normal((n, d))
    R = rot.hd_matrix(hadamard_signs(d, bits))
    err2 = []
    for i in range(n):
        S = rng.standard_normal((d, d))
        comp = qt.compress_prod(x[i:i + 1], R, c, b, S)
        est = att.scores_compressed(y[i:i + 1] * math.sqrt(d), qt.reconstruct_mse(comp.idx, comp.norm, R, c),
                                    comp.rnorm, comp.sigma, S)[0, 0]
        err2.append((est - y[i] @ x[i]) ** 2 / (y[i] @ y[i]))
    dprod = np.mean(err2)
    assert dprod <= math.sqrt(3) * math.pi ** 2 / d * 4.0 ** -bits
    assert dprod >= 1 / d * 4.0 ** -bits


def test_qjl_conditional_variance_bound():
    # Var(<y, x_qjl> | x_mse) <= pi/(2m) ||y||^2 ||r||^2 over fresh S
    rng = np.random.default_rng(27)
    d = 128
    r = rng.standard_normal(d) * 0.05
    y = rng.standard_normal(d)
    vals = []
    for _ in range(5000):
        S = rng.standard_normal((d, d))
        vals.append(y @ qt.qjl_reconstruct((S @ r >= 0)[None], np.array([np.linalg.norm(r)]), S)[0])
    assert np.var(vals) <= math.pi / (2 * d) * (y @ y) * (r @ r)


def test_softmax_attention_matches_torch_sdpa():
    rng = np.random.default_rng(28)
    q = rng.standard_normal((4, 128))
    K = rng.standard_normal((300, 128))
    V = rng.standard_normal((300, 128))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(K)[None], torch.tensor(V)[None])[0].numpy()
    np.testing.assert_allclose(att.softmax_attention(q, K, V), ref, rtol=1e-12, atol=1e-12)
    assert np.all(att.softmax_attention(q, K[:0], V[:0]) == 0)


def _compressed_head(rng, T, bits_k, bits_v, qjl, rotation="hd", scale=1.0):
    d = 128
    K = rng.standard_normal((T, d)) * scale
    V = rng.standard_normal((T, d))
    R = rot.hd_matrix(hadamard_signs(d, 0)) if rotation == "hd" else haar_matrix(d, 3)
    S = qjl_matrix(128, d, 1)
    ck, bk = cb.codebook_f32(bits_k, d)
    cv, bv = cb.codebook_f32(bits_v, d)
    kc = qt.compress_prod(K, R, ck, bk, S) if qjl else qt.compress_mse(K, R, ck, bk)
    vc = qt.compress_mse(V, R, cv, bv)
    return K, V, R, S, (ck, bk, cv, bv), kc, vc


def test_compressed_scores_equal_dense_reconstruction_route():
    # <q,k_mse> + ||r|| sqrt(pi/2)/m <Sq, sign(Sr)> == <q, x_mse + x_qjl>, then SDPA over the
    # dense reconstruction (torch) equals the oracle's attention on those scores
    rng = np.random.default_rng(29)
    K, V, R, S, (ck, bk, cv, bv), kc, vc = _compressed_head(rng, 500, 3, 3, True)
    q = rng.standard_normal((3, 128))
    k_mse = qt.reconstruct_mse(kc.idx, kc.norm, R, ck)
    khat = k_mse + qt.qjl_reconstruct(kc.sigma, kc.rnorm, S)
    sc = att.scores_compressed(q, k_mse, kc.rnorm, kc.sigma, S)
    np.testing.assert_allclose(sc, q @ khat.T / math.sqrt(128), rtol=1e-10, atol=1e-12)
    vhat = qt.reconstruct_mse(vc.idx, vc.norm, R, cv)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(khat)[None], torch.tensor(vhat)[None])[0].numpy()
    np.testing.assert_allclose(att.attend_scores(sc, vhat), ref, rtol=1e-10, atol=1e-12)


def test_pre_rotated_query_identity():
    # <q, R^T c> == <R q, c>: the identity the device path relies on
    rng = np.random.default_rng(30)
    for R in (rot.hd_matrix(hadamard_signs(128, 2)), haar_matrix(128, 2)):
        q = rng.standard_normal(128)
        c = rng.standard_normal(128)
        assert abs(q @ rot.unrotate(R, c[None])[0] - rot.rotate(R, q[None])[0] @ c) < 1e-10


def test_decode_over_packed_pages_equals_dense_route():
    rng = np.random.default_rng(31)
    fmt = lay.Format(key_bits=2, key_qjl=True, value_bits=2)
    T = 700
    K, V, R, S, (ck, bk, cv, bv), kc, vc = _compressed_head(rng, T, 2, 2, True)
    cache = lay.empty_cache(fmt, 4, 1)
    bt = np.array([[3, 1, 0]])
    lay.write_sequence(cache, fmt, 0, 0, bt[0], kc, vc)
    q = rng.standard_normal((1, 2, 1, 128))
    out = att.decode(cache, fmt, 0, q, bt, [T], R, ck, cv, S)
    k_mse = qt.reconstruct_mse(kc.idx, kc.norm, R, ck)
    khat = k_mse + qt.qjl_reconstruct(kc.sigma, kc.rnorm, S)
    vhat = qt.reconstruct_mse(vc.idx, vc.norm, R, cv)
    for h in range(2):
        ref = att.softmax_attention(q[0, h], khat, vhat)
        np.testing.assert_allclose(out[0, h], ref, rtol=1e-10, atol=1e-12)


def test_scores_scaled_by_inverse_sqrt_d():
    rng = np.random.default_rng(32)
    q = rng.standard_normal((1, 128))
    k = rng.standard_normal((5, 128))
    sc = att.scores_compressed(q, k, None, None, None)
    np.testing.assert_allclose(sc, q @ k.T / math.sqrt(128), rtol=1e-14)


def test_argmax_key_recovered_and_scores_correlate():
    # config-1-shaped data: N(0,1) keys with 4 outlier channels x8, 2-bit + QJL keys
    rng = np.random.default_rng(33)
    d, T = 128, 4096
    K = rng.standard_normal((T, d))
    oc = np.random.default_rng(3).choice(d, 4, replace=False)
    K[:, oc] *= 8
    q = rng.standard_normal(d)
    K[1234] = 2.0 * q + 0.3 * rng.standard_normal(d)
    R = rot.hd_matrix(hadamard_signs(d, 0))
    S = qjl_matrix(128, d, 1)
    ck, bk = cb.codebook_f32(2, d)
    kc = qt.compress_prod(K, R, ck, bk, S)
    k_mse = qt.reconstruct_mse(kc.idx, kc.norm, R, ck)
    est = att.scores_compressed(q[None], k_mse, kc.rnorm, kc.sigma, S)[0]
    true = K @ q / math.sqrt(d)
    assert np.argmax(est) == np.argmax(true) == 1234
    assert np.corrcoef(est, true)[0, 1] > 0.9


def test_more_bits_lower_score_error():
    rng = np.random.default_rng(34)
    prev = np.inf
    q = rng.standard_normal((4, 128))
    for bits in (2, 3, 4):
        K, V, R, S, (ck, bk, cv, bv), kc, vc = _compressed_head(rng, 2000, bits, 2, True)
        k_mse = qt.reconstruct_mse(kc.idx, kc.norm, R, ck)
        est = att.scores_compressed(q, k_mse, kc.rnorm, kc.sigma, S)
        err = np.mean((est - q @ K.T / math.sqrt(128)) ** 2)
        assert err < prev
        prev = err


def test_value_qjl_decode_is_unbiased_where_mse_only_is_not():
    # Values with QJL ("TurboQuant explained", section "Two-Stage Approach": x_mse + x_qjl is
    # an unbiased reconstruction, so TurboQuant_prod serves the value cache too).  With all
    # keys equal the softmax weights are uniform, so the decode output is the mean of the
    # reconstructed values: over fresh S its average must reach mean_t v_t, while the
    # MSE-only decode keeps the 1-bit quantiser's shrinkage.  A wrong sign, scale or
    # orientation of the value QJL term in the decode fails this.
    rng = np.random.default_rng(31)
    d, T, trials = 64, 6, 3000
    R = rot.hd_matrix(hadamard_signs(d, 4))
    ck, kb = cb.codebook_f32(2, d)
    cv, vb = cb.codebook_f32(1, d)
    V = rng.standard_normal((T, d)) * 3.0
    K = np.tile(rng.standard_normal(d), (T, 1))
    q = rng.standard_normal((1, d))
    kc = qt.compress_mse(K, R, ck, kb)
    target = V.mean(axis=0)
    acc_q = np.zeros(d)
    acc_m = np.zeros(d)
    for _ in range(trials):
        S = rng.standard_normal((d, d))
        vc = qt.compress_prod(V, R, cv, vb, S)
        u = lay.Unpacked(k_idx=kc.idx, k_norm=kc.norm, v_idx=vc.idx, v_norm=vc.norm,
                         v_rnorm=vc.rnorm, v_sigma=vc.sigma)
        acc_q += att.decode_sequence(q, u, R, ck, cv, S)[0]
        u.v_rnorm = u.v_sigma = None
        acc_m += att.decode_sequence(q, u, R, ck, cv, S)[0]
    err_q = np.linalg.norm(acc_q / trials - target)
    err_m = np.linalg.norm(acc_m / trials - target)
    assert err_m > 0.15 * np.linalg.norm(target)       # the MSE-only output is biased
    assert err_q < 0.25 * err_m                        # the QJL term removes the bias
    assert err_q < 0.05 * np.linalg.norm(target)


def test_value_qjl_single_token_output_is_the_prod_reconstruction():
    # one cached token: softmax weight 1, so decode returns that token's v_mse + x_qjl
    rng = np.random.default_rng(32)
    d = 128
    R = rot.hd_matrix(hadamard_signs(d, 0))
    S = qjl_matrix(128, d, 1)
    ck, kb = cb.codebook_f32(3, d)
    cv, vb = cb.codebook_f32(2, d)
    k = rng.standard_normal((1, d))
    v = rng.standard_normal((1, d))
    kc = qt.compress_prod(k, R, ck, kb, S)
    vc = qt.compress_prod(v, R, cv, vb, S)
    u = lay.Unpacked(k_idx=kc.idx, k_norm=kc.norm, v_idx=vc.idx, v_norm=vc.norm, k_rnorm=kc.rnorm,
                     k_sigma=kc.sigma, v_rnorm=vc.rnorm, v_sigma=vc.sigma)
    out = att.decode_sequence(rng.standard_normal((2, d)), u, R, ck, cv, S)
    r = v[0] - qt.reconstruct_mse(vc.idx, vc.norm, R, cv)[0]
    expect = qt.reconstruct_mse(vc.idx, vc.norm, R, cv)[0] + \
        math.sqrt(math.pi / 2) / 128 * vc.rnorm[0] * (S.T @ np.where(S @ r >= 0, 1.0, -1.0))
    np.testing.assert_allclose(out, np.tile(expect, (2, 1)), rtol=1e-12, atol=1e-12)
