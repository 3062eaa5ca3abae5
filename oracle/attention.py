"""Inner-product estimators and decode attention (oracle; test infrastructure).

Sources:
  * "TurboQuant explained" (Mobilint blog):
      - section "The KV Cache Problem": attention scores are inner products of
        the current query with every cached key, followed by softmax (the
        1/sqrt(d_k) factor is restored here);
      - section "QJL: Inner Product Recovery from a Single Sign Bit": the
        estimator <q,k>^ = sqrt(pi/2)/m * ||k|| * <S q, sign(S k)>, unbiased;
      - section "Two-Stage Approach: MSE Approximation + QJL Correction" and
        "Unbiasedness Proof": the key is x_mse + x_qjl, so
        <q, k>^ = <q, k_mse> + ||r|| sqrt(pi/2)/m <S q, sign(S r)>;
      - the same section, on the value cache: a vector is reconstructed as
        x_mse + sqrt(pi/2)/d ||r|| S^T sign(S r), unbiased, so TurboQuant_prod serves the
        value cache as well (values with QJL);
      - section "How is this different from PolarQuant's reconstruction?": the
        identity <q, R^T c> = <R q, c>, which the device path uses; this oracle
        computes <q, k_mse> directly in the original space instead.
  * "turboquant_cutile" function list: "Asymmetric estimator: term1 (MSE dot) +
    term2 (QJL correction)"; "Full pipeline: scores -> softmax -> weighted V
    sum"; "Scores should be scaled by 1/sqrt(d)"; the decode case seq_q = 1.

Readings taken where the pages are open:
  * grouped-query attention: query head h reads kv head floor(h / G), G = q_heads / kv_heads;
  * every query position of a block sees the whole cached sequence (no causal mask);
  * an empty sequence gives an all-zero output;
  * m (rows of S) divides the QJL sum; m = d in every configuration.
"""
from __future__ import annotations

import math

import numpy as np

from . import layout as lay
from . import quant as qt
from . import rotation as rot


def qjl_estimate(q, k, S) -> float:
    """sqrt(pi/2)/m * ||k|| * <S q, sign(S k)> for one pair (sign(0) taken as +1)."""
    S = np.asarray(S, dtype=np.float64)
    m = S.shape[0]
    sk = S @ np.asarray(k, dtype=np.float64)
    sgn = np.where(sk >= 0, 1.0, -1.0)
    return math.sqrt(math.pi / 2.0) / m * np.linalg.norm(k) * float((S @ q) @ sgn)


def softmax_attention(q, K, V) -> np.ndarray:
    """softmax(q K^T / sqrt(d)) V for q [nq, d], K, V [T, d] (T may be 0)."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros((q.shape[0], V.shape[1]))
    s = q @ K.T / math.sqrt(q.shape[1])
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ V


def scores_compressed(q, k_mse, rnorm, sigma, S) -> np.ndarray:
    """Asymmetric scores for q [nq, d] against compressed keys:
    (<q, k_mse> + ||r|| sqrt(pi/2)/m <S q, 2 sigma - 1>) / sqrt(d).  rnorm/sigma None = MSE only."""
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[1]
    s = q @ np.asarray(k_mse, dtype=np.float64).T
    if sigma is not None:
        S = np.asarray(S, dtype=np.float64)
        m = S.shape[0]
        pm = np.where(np.asarray(sigma), 1.0, -1.0)
        s = s + math.sqrt(math.pi / 2.0) / m * ((q @ S.T) @ pm.T) * np.asarray(rnorm)[None, :]
    return s / math.sqrt(d)


def attend_scores(scores, Vhat) -> np.ndarray:
    """softmax over the token axis of precomputed scores, then the weighted sum of Vhat."""
    if scores.shape[1] == 0:
        return np.zeros((scores.shape[0], Vhat.shape[1]))
    s = scores - scores.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ Vhat


def decode_sequence(q, unpacked: lay.Unpacked, R, ck, cv, S=None, return_scores=False):
    """Decode attention of q [nq, d] over one (sequence, kv head) read from packed pages.
    Values with QJL are reconstructed as v_mse + x_qjl (S is then required); dithered
    vectors add their stored offset back before un-rotating."""
    k_mse = qt.reconstruct_mse(unpacked.k_idx, unpacked.k_norm, R, ck, unpacked.k_offset)
    v_hat = qt.reconstruct_mse(unpacked.v_idx, unpacked.v_norm, R, cv, unpacked.v_offset)
    if unpacked.v_sigma is not None:
        v_hat = v_hat + qt.qjl_reconstruct(unpacked.v_sigma, unpacked.v_rnorm, S)
    sc = scores_compressed(q, k_mse, unpacked.k_rnorm, unpacked.k_sigma, S)
    out = attend_scores(sc, v_hat)
    return (out, sc) if return_scores else out


def decode(cache, fmt: lay.Format, layer: int, q, block_table, seq_lens, R, ck, cv, S=None,
           heads=None):
    """Decode attention for q [B][Hq][seq_q][d] over a packed cache [L][pages][Hkv][block].

    heads (optional): list of (b, h) query-head pairs to compute; others stay 0."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, sq, d = q.shape
    Hkv = cache.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, Hq, sq, d))
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    cache_unpacked = {}
    for (b, h) in todo:
        kvh = h // G
        key = (b, kvh)
        if key not in cache_unpacked:
            n = int(seq_lens[b])
            cache_unpacked[key] = lay.read_sequence(cache, fmt, layer, kvh, block_table[b], n)
        out[b, h] = decode_sequence(q[b, h], cache_unpacked[key], R, ck, cv, S)
    return out
