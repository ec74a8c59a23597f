"""Pins of the oracle's integer-range report and of the weights path's dither counter.

The range report follows the pages' integer implementation (explainer pages,
"Methodology" 2): the lattice points' integers are meant to fit 8-bit storage,
with alpha calibrated so that they do not overflow.  Reading R11: the Rice code
is unbounded, nothing is clamped, and the encoder reports the largest |code
coordinate| and the number of coordinates outside [-128, 127].

The closed-form cases use inputs whose transformed tile is known exactly: with
alpha = fp32(sqrt(128)) the forward scale fp32(alpha / sqrt(128)) is exactly 1,
and the unnormalised Sylvester H_128 maps a one-hot input at column 0 to a
constant vector (its first column is all ones) and the pair (columns 0, 1) with
equal signed values to (2t, 0, 2t, 0, ...).  Those vectors are lattice points of
Z, D4 and 2E8 themselves (and of A2 in its (a, b) code form), so the codes are
known without running a decoder.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth

ALPHA_UNIT = float(np.float32(np.sqrt(128.0)))   # forward scale exactly 1


def test_unit_alpha_gives_unit_scale():
    assert np.float32(np.float64(np.float32(ALPHA_UNIT)) / np.sqrt(128.0)) == np.float32(1.0)
    assert O.scale_fwd(ALPHA_UNIT) == 1.0


def test_code_range_definition():
    """Largest |q| and the count outside int8, on hand-written codes."""
    assert O.code_range([]) == (0, 0)
    assert O.code_range([0, 0, 0]) == (0, 0)
    assert O.code_range([-128, 127, 3, -7]) == (128, 0)        # both ends of int8 fit
    assert O.code_range([128]) == (128, 1)
    assert O.code_range([-129]) == (129, 1)
    assert O.code_range([127, 128, -128, -129, 200, -5]) == (200, 3)
    assert O.code_range([1 << 20, -(1 << 20) - 3]) == ((1 << 20) + 3, 2)


def _one_hot_rows(values):
    """A matrix of len(values) rows x 256 columns: row r holds values[r] at column 0."""
    x = torch.zeros(len(values), 256, dtype=torch.float32)
    x[:, 0] = torch.tensor(values, dtype=torch.float32)
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("lat", [O.Z, O.D4, O.E8])
def test_range_of_constant_tiles_is_closed_form(lat):
    """One-hot rows at column 0: every code coordinate of the row's first tile is
    s_0 * value (s_0 the sign of column 0), every other code is 0."""
    seed = 3
    s0 = O.sign(seed, 0)
    values = [5.0, -5.0, 127.0, -127.0, 128.0, -128.0, 129.0, -129.0, 200.0, -200.0]
    for v in values:
        x = _one_hot_rows([v])
        t = int(s0 * v)
        mx, ov = O.quantize_range(x, lat, ALPHA_UNIT, seed)
        assert mx == abs(t), (lat, v)
        assert ov == (128 if (t < -128 or t > 127) else 0), (lat, v)
    # a matrix of several such rows: the maximum and the sum over rows
    x = _one_hot_rows(values)
    mx, ov = O.quantize_range(x, lat, ALPHA_UNIT, seed)
    assert mx == 200
    assert ov == 128 * sum(1 for v in values if not (-128 <= int(s0 * v) <= 127))


@pytest.mark.parametrize("lat,factor", [(O.Z, 2), (O.D4, 2), (O.E8, 2), (O.A2, 4)])
def test_range_of_alternating_tiles_is_closed_form(lat, factor):
    """Columns 0 and 1 set so that s_0 x_0 = s_1 x_1 = t: the tile becomes
    (2t, 0, 2t, 0, ...).  Z, D4 and 2E8 code it as itself (largest |code| 2|t|);
    A2 codes each pair (2t, 0) as (a, b) = (4t, 0), the point (a/2, b sqrt(3)/2)."""
    seed = 11
    s0, s1 = O.sign(seed, 0), O.sign(seed, 1)
    for t in (3, -3, 31, -32, 32, 64, -64, 65):
        x = torch.zeros(1, 128, dtype=torch.float32)
        x[0, 0] = s0 * t
        x[0, 1] = s1 * t
        x = x.to(torch.bfloat16)
        mx, ov = O.quantize_range(x, lat, ALPHA_UNIT, seed)
        big = factor * t
        assert mx == abs(big), (lat, t)
        assert ov == (64 if not (-128 <= big <= 127) else 0), (lat, t)   # half of the coordinates


def test_range_matches_the_codes_of_the_stream():
    """On ordinary data the range is that of the integer codes the stream carries:
    decode every chunk of the oracle's own stream back to codes and take the range
    of those (the chunk coder is pinned by the round-trip and textbook-codeword pins)."""
    x = synth.weight(48, 512, seed=7)
    for lat, alpha in ((O.E8, 3000.0), (O.D4, 2000.0), (O.A2, 2500.0), (O.Z, 2000.0)):
        s, off, _ = O.quantize(x, lat, alpha, 3, 5)
        codes = []
        nch = O.n_chunks(48, 512)
        for c in range(nch):
            nt = min(32, 48 * 4 - 32 * c)
            codes.append(O.decode_chunk(lat, 3, s[int(off[c]):int(off[c + 1])], nt))
        q = np.concatenate(codes)
        want = (int(np.abs(q.astype(np.int64)).max()), int(((q < -128) | (q > 127)).sum()))
        assert O.quantize_range(x, lat, alpha, 5) == want
        assert want[1] > 0        # the case reaches past int8


def test_weights_dither_counter_is_row_major_element_index():
    """With dither, weight tile (r, tc) is coded at dither counter r * C + 128 tc (the
    element index of its first element): the stream's codes equal the tile quantizer's
    at exactly that counter, and not at a neighbouring one."""
    R, C = 5, 384
    x = synth.weight(R, C, seed=12)
    xu = x.view(torch.int16).numpy().view(np.uint16)
    alpha, k, seed = 250.0, 2, 23
    for lat in (O.E8, O.Z):
        s, off, _ = O.quantize(x, lat, alpha, k, seed, dither=1)
        q = O.decode_chunk(lat, k, s[int(off[0]):int(off[1])], R * C // 128)
        for r in range(R):
            for tc in range(C // 128):
                i = r * (C // 128) + tc
                got = q[i * 128:(i + 1) * 128]
                want = O.quantize_tile(xu[r, 128 * tc:128 * (tc + 1)], lat, alpha, seed, sign_col0=128 * tc,
                                       dither=1, e0=r * C + 128 * tc)
                assert np.array_equal(got, want), (lat, r, tc)
        # a shifted counter gives other codes (the counter is used)
        other = O.quantize_tile(xu[1, 128:256], lat, alpha, seed, sign_col0=128, dither=1, e0=1 * C + 128 + 128)
        assert not np.array_equal(q[4 * 128:5 * 128], other)
