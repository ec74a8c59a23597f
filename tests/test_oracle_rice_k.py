"""Pins of the per-position Rice parameter (CPU only).

Bit-stripping halves the last symbol of each A2, D4 and E8 block (b', q3', m7': the
implied parity bit is removed), so that symbol is about half the size of the others
and its best Rice parameter is smaller.  With `dk_last` > 0 it is coded with
max(k - dk_last, 0) and every other symbol with k; dk_last = 0 is the single-k code.
These tests pin the oracle's chunk coder in that mode against the textbook Rice code
with a parameter per symbol (the planes must hold exactly those codeword bits),
against the definition of which symbol is the last one, and against the fact that
the mode changes only the bitstream, never the codes or the reconstruction.
"""
import math

import numpy as np
import pytest

import oracle as O
import synth

LAST = {O.Z: None, O.A2: 1, O.D4: 3, O.E8: 7}


def _ks(lat, k, dk, nsym):
    n = O.DIM[lat]
    return [max(k - dk, 0) if (LAST[lat] is not None and i % n == LAST[lat]) else k for i in range(nsym)]


def _bits(words, n):
    return [(int(words[j >> 5]) >> (j & 31)) & 1 for j in range(n)]


def test_symbol_k_follows_the_definition():
    for lat in (O.Z, O.A2, O.D4, O.E8):
        for k in range(16):
            for dk in range(5):
                assert [O.symbol_k(lat, k, dk, i) for i in range(O.DIM[lat])] == _ks(lat, k, dk, O.DIM[lat])


def test_per_symbol_rice_concat_is_the_textbook_code():
    # z = 9 with k = 2: two zeros, a one, remainder 01; z = 3 with k = 0: three zeros and a one
    words, nbits = O.rice_concat_k(np.array([9, 3], np.uint32), np.array([2, 0], np.int32))
    assert nbits == 5 + 4
    assert _bits(words, nbits) == [0, 0, 1, 1, 0] + [0, 0, 0, 1]
    z = np.random.default_rng(1).geometric(0.2, 300).astype(np.uint32)
    for k in (0, 3):
        assert np.array_equal(O.rice_concat_k(z, np.full(300, k, np.int32))[0], O.rice_concat(z, k)[0])


@pytest.mark.parametrize("lat", [O.Z, O.A2, O.D4, O.E8])
@pytest.mark.parametrize("k,dk", [(0, 1), (2, 1), (2, 2), (5, 1), (5, 3)])
def test_two_k_planes_hold_the_textbook_codewords(lat, k, dk):
    rng = np.random.default_rng(70 + lat * 11 + k * 3 + dk)
    n = O.DIM[lat]
    for ntiles in (1, 3, 32):
        v = (rng.normal(size=ntiles * 128) * rng.choice([0.5, 4.0, 30.0])).astype(np.float32)
        v[::89] *= 40
        q = np.concatenate([O.decode(lat, v[i:i + n]) for i in range(0, len(v), n)])
        words, payload = O.encode_chunk(lat, k, q, dk)
        assert np.array_equal(O.decode_chunk(lat, k, words, ntiles, dk), q)
        syms, nblk = [], len(q) // n
        for b in range(0, len(q), n):
            m, _ = O.strip(lat, q[b:b + n])
            syms += [O.zigzag(int(x)) for x in m]
        ks = _ks(lat, k, dk, len(syms))
        cat, nbits = O.rice_concat_k(np.array(syms, np.uint32), np.array(ks, np.int32))
        assert payload == nbits + (nblk if lat == O.E8 else 0)
        # rebuild the concatenated codewords from the planes: unary runs and remainder fields in order
        nc = math.ceil(nblk / 32) if lat == O.E8 else 0
        nr = math.ceil(sum(ks) / 32)
        rem = _bits(words[nc:nc + nr], 32 * nr)
        un = _bits(words[nc + nr:], 32 * (len(words) - nc - nr))
        rebuilt, rp, up = [], 0, 0
        for i in range(len(syms)):
            while un[up] == 0:
                rebuilt.append(0)
                up += 1
            rebuilt.append(1)
            up += 1
            rebuilt += rem[rp:rp + ks[i]]
            rp += ks[i]
        assert rebuilt == _bits(cat, nbits)
        assert not any(un[up:]) and not any(rem[rp:])      # the plane tails are zero padding


@pytest.mark.parametrize("lat,alpha", [(O.A2, 130.0), (O.D4, 183.8), (O.E8, 314.15)])
def test_two_k_changes_only_the_bitstream(lat, alpha):
    """The same codes and reconstruction; fewer bits, since the halved symbol is about
    half the size of the others (near 4 bits per scalar here)."""
    x = synth.weight(16, 1024, seed=5)
    s0, off0, p0 = O.quantize(x, lat, alpha, 2, 3)
    s1, off1, p1 = O.quantize(x, lat, alpha, 2, 3, dk_last=1)
    y0 = O.dequantize(s0, off0, 16, 1024, lat, alpha, 2, 3, out_fp32=True)
    y1 = O.dequantize(s1, off1, 16, 1024, lat, alpha, 2, 3, out_fp32=True, dk_last=1)
    assert np.array_equal(y0, y1)
    assert p1 < p0
    K, _ = synth.kv(2, 40, seed=3)
    a, offa, _ = O.kv_append(K, 0, lat, 1.0, 1, 7, 1)
    b, offb, _ = O.kv_append(K, 0, lat, 1.0, 1, 7, 1, dk_last=1)
    ya = np.zeros((2, 40, 128), np.float32)
    yb = np.zeros((2, 40, 128), np.float32)
    O.kv_read_append(a, offa, 2, 40, 0, lat, 1.0, 1, 7, 1, ya, 40)
    O.kv_read_append(b, offb, 2, 40, 0, lat, 1.0, 1, 7, 1, yb, 40, dk_last=1)
    assert np.array_equal(ya, yb)
