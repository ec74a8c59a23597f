"""Pins of the oracle's dense KV rotation (CPU only).

The explainer pages ("Methodology" 4) rotate each layer's keys and values either by
the cheap sign diagonal (with H_128, the default path) or by a full Haar-uniform
matrix.  These tests pin the Haar variant against facts the oracle does not compute:
the normal distribution (Kolmogorov-Smirnov), the uniqueness of QR with a positive
diagonal, the trace moments of Haar-distributed orthogonal matrices (Diaconis and
Shahshahani), exact single-term sums, orthogonality, and the unbiasedness that
subtractive dither gives whatever the rotation is.
"""
import math

import numpy as np
import pytest
import scipy.stats
import torch

import oracle as O
from oracle import rotation as R
import synth


def test_gaussian_draws_are_standard_normal():
    g = np.array([O.rot_gaussian(3, e) for e in range(40000)])
    assert scipy.stats.kstest(g, "norm").pvalue > 1e-3
    assert abs(g.mean()) < 4 / math.sqrt(g.size)
    assert abs(g.var() - 1.0) < 4 * math.sqrt(2.0 / g.size)
    # the draws of another seed are another sequence
    h = np.array([O.rot_gaussian(4, e) for e in range(200)])
    assert not np.allclose(g[:200], h)


def test_haar_matrix_is_orthogonal_in_fp32():
    for seed in (0, 1, 77):
        Q = R.haar_rotation(seed).astype(np.float64)
        # exact orthogonal matrix rounded once to fp32: |Q^T Q - I| <= 2 * 2^-24 * max row norm^2
        assert np.abs(Q.T @ Q - np.eye(128)).max() < 2.5 * 2.0**-24 * 1.0 + 1e-7
        assert np.abs(Q @ Q.T - np.eye(128)).max() < 1e-6


def test_haar_matrix_is_the_positive_diagonal_qr_factor():
    """G = Q R with R upper triangular and positive on its diagonal (unique); its first
    column is therefore G's first column normalised (the first Gram-Schmidt step)."""
    for seed in (2, 5):
        G = R.gaussian_matrix(seed)
        Q, _ = R.haar_rotation_f64(seed)
        Rm = Q.T @ G
        assert np.abs(np.tril(Rm, -1)).max() < 1e-11 * np.abs(G).max()
        assert np.all(np.diag(Rm) > 0)
        assert np.allclose(Q[:, 0], G[:, 0] / np.linalg.norm(G[:, 0]), rtol=0, atol=1e-14)
        assert np.array_equal(R.haar_rotation(seed), Q.astype(np.float32))


def test_haar_trace_moments():
    """For Haar-distributed Q in O(n), n large, tr Q has mean 0 and variance 1 and tr Q^2
    has mean 1 (Diaconis-Shahshahani).  Without the sign correction the QR factor is not
    Haar: its trace averages about -6.5 here, so this pin has power."""
    t1, t2 = [], []
    for seed in range(200):
        Q = R.haar_rotation(1000 + seed).astype(np.float64)
        t1.append(np.trace(Q))
        t2.append(np.trace(Q @ Q))
    t1, t2 = np.array(t1), np.array(t2)
    n = len(t1)
    assert abs(t1.mean()) < 4 / math.sqrt(n)
    assert 0.65 < t1.var() < 1.45
    assert abs(t2.mean() - 1.0) < 4 * math.sqrt(2.0 / n)


def test_rotation_of_basis_vectors_is_exact():
    """One nonzero term: forward of e_j is column j of Q, inverse of e_i is row i."""
    Q = R.haar_rotation(9)
    for j in (0, 1, 63, 127):
        e = np.zeros(128, np.float32)
        e[j] = 1.0
        assert np.array_equal(O.rotate_fwd(Q, e), Q[:, j])
        assert np.array_equal(O.rotate_inv(Q, e), Q[j, :])
        e[j] = -0.375
        assert np.array_equal(O.rotate_fwd(Q, e), (Q[:, j] * np.float32(-0.375)).astype(np.float32))


def test_rotation_sums_within_fp32_bound_and_round_trip():
    Q = R.haar_rotation(10)
    Q64 = Q.astype(np.float64)
    rng = np.random.default_rng(5)
    u = 2.0**-24
    for scale in (1e-3, 1.0, 1e3):
        x = (rng.normal(size=128) * scale).astype(np.float32)
        y = O.rotate_fwd(Q, x).astype(np.float64)
        exact = Q64 @ x.astype(np.float64)
        bound = 128 * u * (np.abs(Q64) @ np.abs(x.astype(np.float64)))
        assert np.all(np.abs(y - exact) <= bound)
        back = O.rotate_inv(Q, y.astype(np.float32)).astype(np.float64)
        assert np.abs(back - x).max() < 1e-5 * np.abs(x).max()


@pytest.mark.parametrize("lat", [O.Z, O.A2, O.D4, O.E8])
def test_rotated_roundtrip_error_within_covering_bound(lat):
    """Q is orthogonal, so per tile ||x_hat - x||^2 <= blocks * r^2 / alpha^2 (up to the
    fp32 rounding of Q), the same bound as with H_128 D."""
    Q = R.haar_rotation(11)
    K, _ = synth.kv(2, 40, seed=6)
    alpha = 6.0
    s, off, _ = O.kv_append(K, 0, lat, alpha, 1, 3, dither=0, rot=Q)
    out = np.zeros((2, 40, 128), np.float32)
    O.kv_read_append(s, off, 2, 40, 0, lat, alpha, 1, 3, 0, out, 40, rot=Q)
    r2 = {O.Z: 0.25, O.A2: 1 / 3, O.D4: 1.0, O.E8: 4.0}[lat]
    err = ((out.astype(np.float64) - K.float().numpy()) ** 2).sum(-1)
    assert err.max() <= (128 // O.DIM[lat]) * r2 / alpha**2 * (1 + 1e-3) + 1e-9


def test_rotated_dithered_reconstruction_is_unbiased_regression():
    """With subtractive dither the error is independent of the input: the least-squares
    slope of x_hat on x is 1 only if the forward and inverse rotation and scales agree."""
    Q = R.haar_rotation(12)
    K, _ = synth.kv(4, 512, seed=7)
    alpha = 1.2
    s, off, _ = O.kv_append(K, 0, O.E8, alpha, 1, 21, dither=1, rot=Q)
    y = np.zeros((4, 512, 128), np.float32)
    O.kv_read_append(s, off, 4, 512, 0, O.E8, alpha, 1, 21, 1, y, 512, rot=Q)
    y = y.astype(np.float64)
    xf = K.float().numpy().astype(np.float64)
    slope = float((y * xf).sum() / (xf * xf).sum())
    resid = y - xf
    se = float(resid.std() / (xf.std() * math.sqrt(xf.size)))
    assert abs(slope - 1.0) < 5 * se, (slope, se)
    assert abs(float(np.corrcoef(resid.reshape(-1), xf.reshape(-1))[0, 1])) < 5 / math.sqrt(xf.size)


def test_rotated_append_tiles_match_the_tile_functions():
    """The KV append with a rotation codes every token's head vector with the rotated
    tile quantizer at its dither counter, and reads back with the rotated inverse."""
    Q = R.haar_rotation(13)
    K, _ = synth.kv(3, 37, seed=8)
    ku = K.view(torch.int16).numpy().view(np.uint16)
    tok0, alpha, k, seed = 5, 0.9, 1, 17
    s, off, _ = O.kv_append(K, tok0, O.D4, alpha, k, seed, dither=1, rot=Q)
    out = np.zeros((3, tok0 + 37, 128), np.float32)
    O.kv_read_append(s, off, 3, 37, tok0, O.D4, alpha, k, seed, 1, out, tok0 + 37, rot=Q)
    cph = (37 + 31) // 32
    for h in range(3):
        for t in (0, 31, 32, 36):
            c, i = h * cph + t // 32, t % 32
            nt = min(32, 37 - 32 * (t // 32))
            codes = O.decode_chunk(O.D4, k, s[int(off[c] - off[0]):int(off[c + 1] - off[0])], nt)[i * 128:(i + 1) * 128]
            e0 = ((tok0 + t) * 3 + h) * 128
            assert np.array_equal(codes, O.quantize_tile_rot(ku[h, t], O.D4, alpha, Q, seed, 1, e0))
            assert np.array_equal(out[h, tok0 + t], O.dequantize_tile_rot(codes, O.D4, alpha, Q, seed, 1, e0))
    # the rotation changes the codes (it is used), and the default path is untouched
    s0, _, _ = O.kv_append(K, tok0, O.D4, alpha, k, seed, dither=1)
    assert not np.array_equal(s0, s)
