"""Haar-uniform rotation of the KV path, generated the plain way (test infrastructure).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the tests, the smoke check
and the benchmark's CPU leg use it; the product library has its own generator.

The explainer pages ("Methodology" 4) give each layer's keys and values a random
rotation: a full Haar-uniform matrix, or the cheap sign diagonal.  They do not say
how the Haar matrix is drawn.  Reading [R18]: the Q factor of the QR decomposition
of a 128 x 128 matrix G of independent standard normals, with the signs of its
columns chosen so that R has a positive diagonal.  That factor is Haar-distributed
on O(128) (Mezzadri, "How to generate random matrices from the classical compact
groups", 2007), and it is unique, so any QR method gives the same matrix up to
rounding.  G[i][j] is Gaussian draw 128 i + j of ``hqref_rot_gaussian``.  Q is
computed in double and rounded to fp32 once; the codec uses the fp32 matrix.
"""
from __future__ import annotations

import numpy as np

from . import rot_gaussian

N = 128


def gaussian_matrix(seed: int) -> np.ndarray:
    """G[i][j] = Gaussian draw 128 i + j for this seed, float64 [128, 128]."""
    g = np.empty(N * N, dtype=np.float64)
    for e in range(N * N):
        g[e] = rot_gaussian(seed, e)
    return g.reshape(N, N)


def haar_rotation_f64(seed: int) -> tuple[np.ndarray, np.ndarray]:
    """(Q, R) with G = Q R, Q orthogonal and R upper triangular with R[i][i] > 0."""
    G = gaussian_matrix(seed)
    Q, R = np.linalg.qr(G)                 # LAPACK Householder QR (a library primitive)
    s = np.where(np.diag(R) < 0, -1.0, 1.0)
    return Q * s[None, :], R * s[:, None]


def haar_rotation(seed: int) -> np.ndarray:
    """The rotation the codec uses: fp32 [128, 128], row-major Q[i][j]."""
    return haar_rotation_f64(seed)[0].astype(np.float32)
