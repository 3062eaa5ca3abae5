"""Per-vector TurboQuant compression (oracle; test infrastructure).

Sources:
  * "turboquant_cutile" function list: compress K gives an MSE part plus a 1-bit
    QJL correction (2-bit MSE + 1-bit QJL, 3-bit MSE + 1-bit QJL); compress V is
    MSE-only; decompression is "indices -> centroids -> un-rotate -> rescale".
  * "TurboQuant explained" (Mobilint blog):
      - section "Coordinates Become Predictable After Rotation": the quantizer
        works on the unit vector x/||x|| after a random rotation;
      - section "Designing the Optimal Codebook Without Data", step 1: a value is
        assigned to its nearest centroid, which is the cell between adjacent
        midpoints;
      - section "Two-Stage Approach: MSE Approximation + QJL Correction":
        x_mse = DeQuant(Quant(x)), r = x - x_mse, and the 1-bit stage stores
        sign(S r) with ||r||;
      - section "QJL: Inner Product Recovery from a Single Sign Bit": per token
        the sketch stores m sign bits plus a 16-bit norm.

Readings taken where the pages are open:
  * index = number of boundaries strictly below the value, so a value equal to a
    boundary goes to the lower cell;
  * norms (||x|| and ||r||) are stored as IEEE fp16, round to nearest even; a
    norm that overflows fp16 is an error;
  * the residual is taken against the reconstruction with the *stored* fp16
    norm, so the sketch corrects what the decoder sees;
  * sign(0) is stored as +1 (bit 1): sigma_i = [(S r)_i >= 0];
  * a zero vector has u = 0 (its stored norm 0 makes its reconstruction 0).

Dithered quantization ("Minimum Distortion Quantization with Specified Output
Distribution" page, third abstract: after HD, a random scalar offset is subtracted
before quantizing).  Readings:
  * one offset xi per vector, drawn by the caller (uniform on [-delta/2, delta/2) for
    the uniform grid of oracle.codebook.dither_codebook_f32) and passed in; the method
    uses and stores fp16(xi) (RNE), the 16 bits the pages give every per-token scalar;
  * idx = Quant(y - xi), reconstruction n R^T (c[idx] + xi); for keys with QJL the
    residual is taken against this reconstruction.

Corrected norm ("tq-kv" crate documentation: compress_single_key returns the packed
indices and a "corrected_norm").  Reading: the stored norm is n / ||y_hat|| with y_hat
the dequantized rotated vector (c[idx], plus xi when dithered), so that the
reconstruction n_c R^T y_hat has exactly the input's norm; 0 when y_hat = 0.  The
decoder is unchanged (it scales by whatever norm is stored).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

from . import rotation as rot


class NormOverflow(ValueError):
    pass


def fp16_round(x) -> np.ndarray:
    """Round to the nearest fp16 value (RNE), returned as float64; overflow raises."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore"):
        h = x.astype(np.float16)
    if not np.all(np.isfinite(h)):
        raise NormOverflow("norm does not fit in fp16")
    return h.astype(np.float64)


def quantize(y, boundaries) -> np.ndarray:
    """idx = #{i : beta_i < y} for every coordinate (boundaries promoted to float64)."""
    b = np.asarray(boundaries, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    return (y[..., None] > b).sum(axis=-1).astype(np.int64)


def dequantize(idx, centroids) -> np.ndarray:
    return np.asarray(centroids, dtype=np.float64)[np.asarray(idx)]


def fp16_offset(xi) -> np.ndarray:
    """The dither offset as used and stored: fp16 rounding (RNE), as float64."""
    return np.asarray(xi, dtype=np.float64).astype(np.float16).astype(np.float64)


@dataclasses.dataclass
class Compressed:
    idx: np.ndarray            # [N, d] int
    norm: np.ndarray           # [N] stored fp16 norm (float64 values)
    y: np.ndarray              # [N, d] the quantizer's input (rotated unit vector, minus the
                               # offset when dithered), float64, kept for tie analysis
    rnorm: Optional[np.ndarray] = None   # [N] stored fp16 ||r||
    sigma: Optional[np.ndarray] = None   # [N, m] bool, (S r)_i >= 0
    sr: Optional[np.ndarray] = None      # [N, m] S r (float64), kept for tie analysis
    sr_scale: Optional[np.ndarray] = None  # [N, m] sum_j |S_ij r_j|
    offset: Optional[np.ndarray] = None    # [N] dither offset fp16(xi) (float64 values)


def dequantize_dithered(idx, centroids, offset=None) -> np.ndarray:
    """y_hat = c[idx] (+ xi of each row when dithered)."""
    y_hat = dequantize(idx, centroids)
    if offset is not None:
        y_hat = y_hat + np.asarray(offset, dtype=np.float64)[:, None]
    return y_hat


def compress_mse(x, R, centroids, boundaries, offsets=None, corrected_norm=False) -> Compressed:
    """TurboQuant_mse: n = ||x||, u = x/n, y = R u, idx = Quant(y), stored n = fp16(n).
    offsets: per-row dither xi (idx = Quant(y - fp16(xi))); corrected_norm: store
    fp16(n / ||y_hat||) instead of fp16(n)."""
    x = np.asarray(x, dtype=np.float64)
    n = np.linalg.norm(x, axis=-1)
    inv = np.where(n > 0, 1.0 / np.where(n > 0, n, 1.0), 0.0)
    u = x * inv[:, None]
    y = rot.rotate(R, u)
    off = None if offsets is None else fp16_offset(offsets)
    yq = y if off is None else y - off[:, None]
    idx = quantize(yq, boundaries)
    stored = n
    if corrected_norm:
        yn = np.linalg.norm(dequantize_dithered(idx, centroids, off), axis=-1)
        stored = np.where(yn > 0, n / np.where(yn > 0, yn, 1.0), 0.0)
    return Compressed(idx=idx, norm=fp16_round(stored), y=yq, offset=off)


def reconstruct_mse(idx, norm, R, centroids, offset=None) -> np.ndarray:
    """indices -> centroids -> un-rotate -> rescale: x_mse = n * R^T c[idx]
    (n * R^T (c[idx] + xi) when dithered)."""
    y_hat = dequantize_dithered(idx, centroids, offset)
    return np.asarray(norm, dtype=np.float64)[:, None] * rot.unrotate(R, y_hat)


def compress_prod(x, R, centroids, boundaries, S, offsets=None, corrected_norm=False) -> Compressed:
    """TurboQuant_prod (keys, and values with QJL): MSE stage, residual r = x - x_mse,
    sigma = [S r >= 0], ||r||."""
    x = np.asarray(x, dtype=np.float64)
    comp = compress_mse(x, R, centroids, boundaries, offsets, corrected_norm)
    x_mse = reconstruct_mse(comp.idx, comp.norm, R, centroids, comp.offset)
    r = x - x_mse
    S = np.asarray(S, dtype=np.float64)
    sr = r @ S.T
    comp.rnorm = fp16_round(np.linalg.norm(r, axis=-1))
    comp.sigma = sr >= 0.0
    comp.sr = sr
    comp.sr_scale = np.abs(r) @ np.abs(S).T
    return comp


def qjl_reconstruct(sigma, rnorm, S) -> np.ndarray:
    """x_qjl = sqrt(pi/2)/m * ||r|| * S^T (2 sigma - 1)   (TurboQuant_prod dequantization)."""
    S = np.asarray(S, dtype=np.float64)
    m = S.shape[0]
    pm = np.where(np.asarray(sigma), 1.0, -1.0)
    return np.sqrt(np.pi / 2.0) / m * np.asarray(rnorm, dtype=np.float64)[:, None] * (pm @ S)
