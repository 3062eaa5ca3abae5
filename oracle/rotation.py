"""Rotations (oracle; test infrastructure).

Source: "TurboQuant explained" (Mobilint blog), section "How JL Matrices Evolved":
  * D is a diagonal Rademacher matrix (random +-1 entries);
  * H is the Walsh-Hadamard matrix, an orthogonal +-1 matrix defined
    recursively (H_1 = (1), H_2 = (1/sqrt 2)[[1,1],[1,-1]], H_4 = ...), i.e. the
    normalized Sylvester matrix; the sanity check there builds it as
    hadamard(d)/sqrt(d) and applies y = H @ D @ x;
  * TurboQuant uses the HD stage as its random rotation.
Source: "turboquant_cutile" function list and "TurboQuant explained", section
"Two-Stage Approach: MSE Approximation + QJL Correction": the dense option is a
Haar-distributed orthogonal Pi (QR of a Gaussian), applied as Pi @ x and undone
with Pi^T.

The rotation is built here as an explicit d x d matrix R and applied as a plain
matrix product; the device path uses a butterfly transform instead.
"""
from __future__ import annotations

import math

import numpy as np


def sylvester_hadamard(d: int) -> np.ndarray:
    """Normalized Sylvester matrix H[i, j] = (-1)^popcount(i & j) / sqrt(d), d a power of two."""
    if d < 1 or (d & (d - 1)) != 0:
        raise ValueError("d must be a power of two")
    i = np.arange(d)
    parity = np.zeros((d, d), dtype=np.int64)
    x = i[:, None] & i[None, :]
    while np.any(x):
        parity ^= (x & 1)
        x = x >> 1
    return np.where(parity == 1, -1.0, 1.0) / math.sqrt(d)


def hd_matrix(signs) -> np.ndarray:
    """R = H @ diag(D): first flip signs, then mix (y = H D x)."""
    s = np.asarray(signs, dtype=np.float64)
    return sylvester_hadamard(len(s)) * s[None, :]


def rotation_matrix(rotation: int, signs=None, pi=None) -> np.ndarray:
    """The rotation R of a configuration: 0 = randomized Hadamard HD, 1 = dense Pi."""
    if rotation == 0:
        return hd_matrix(signs)
    if rotation == 1:
        return np.asarray(pi, dtype=np.float64)
    raise ValueError("unknown rotation kind")


def rotate(R: np.ndarray, x: np.ndarray) -> np.ndarray:
    """y = R x for each row of x."""
    return np.asarray(x, dtype=np.float64) @ R.T


def unrotate(R: np.ndarray, y: np.ndarray) -> np.ndarray:
    """x = R^T y for each row of y."""
    return np.asarray(y, dtype=np.float64) @ R
