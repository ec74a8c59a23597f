"""The decoder's work split against the oracle, in each of its regimes.

A launch with at least as many chunks as the grid has warps decodes whole chunks per
warp; a shorter one lets two or four warps share a chunk (two rounds or one each).
The grid is at most 3 CTAs of 8 warps per SM without dither, 2 with dither or a second
Rice parameter, and one CTA of 12 warps with the dense KV rotation, so on a 148-SM
B200 the regimes change at 888 / 1776 chunks, 592 / 1184 and 444 / 888.  The sizes
below sit on both sides of every boundary; on another SM count they still span all
three regimes.  Every tile decodes to the oracle's value whichever warp takes it."""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import rotation as R
import synth
from hqtest import assert_recon_equal, gpu_dequantize, oracle_dequantize, oracle_quantize, rate_points, u16

pytestmark = pytest.mark.gpu


def _hq():
    import lattice_entropy_coded_b200 as hq
    return hq


def _alpha(lat, bps=4.0):
    return {p["lattice"]: p["alpha"] for p in rate_points()["weight_4096x4096_rate_sweep"]["points"]
            if p["bps"] == bps}[lat]


def _decode_oracle_stream(rows, cols, lat, k, dither, dk=0, seed=5):
    """GPU decode of the oracle's own stream vs the oracle's decode (fp32)."""
    hq = _hq()
    L = O.LATTICES[lat]
    alpha = _alpha(lat)
    x = synth.weight(rows, cols, seed=rows)
    ref_w, ref_off, _ = oracle_quantize(x, L, alpha, k, seed, dither, dk_last=dk)
    p = hq.make_params(lat, alpha, k, seed, dither, dk_last=dk)
    words = torch.from_numpy(ref_w.view(np.int32).copy()).cuda()
    offs = torch.from_numpy(ref_off.view(np.int64).copy()).cuda()
    y, st, _ = gpu_dequantize(words, len(ref_w), offs, rows, cols, p, fp32=True)
    assert st["status"] == 0
    assert_recon_equal(y, oracle_dequantize(ref_w, ref_off, rows, cols, L, alpha, k, seed, dither, fp32=True,
                                            dk_last=dk))
    return ref_w, ref_off, p


# one chunk per row at 4096 columns
@pytest.mark.parametrize("chunks", [1, 3, 110, 887, 888, 889, 1200, 1776, 1777, 2600, 3552, 3553])
def test_weights_every_regime(chunks):
    _decode_oracle_stream(chunks, 4096, "E8", 2, 0)


@pytest.mark.parametrize("chunks", [591, 592, 593, 1184, 1185, 2400])
@pytest.mark.parametrize("dither,dk", [(1, 0), (0, 1)])
def test_two_cta_regimes(chunks, dither, dk):
    _decode_oracle_stream(chunks, 4096, "D4", 2, dither, dk=dk)


@pytest.mark.parametrize("lat", ["Z", "A2"])
def test_ragged_rows(lat):
    """3556 rows of 1152 columns (9 tiles a row): 1001 chunks, most starting mid-row, the
    last one of 4 tiles; two warps per chunk on a B200."""
    _decode_oracle_stream(3556, 1152, lat, 3, 0)


def test_corrupt_chunk_shared_by_warps():
    """A chunk whose unary plane loses a terminator, in the two-warps-per-chunk regime:
    the call reports it, and every other chunk still decodes to the oracle's values."""
    hq = _hq()
    rows, cols = 1200, 4096
    ref_w, ref_off, p = _decode_oracle_stream(rows, cols, "E8", 2, 0)
    bad = 700
    w = ref_w.copy()
    w[int(ref_off[bad + 1]) - 1] = 0          # the last unary word of chunk 700
    words = torch.from_numpy(w.view(np.int32).copy()).cuda()
    offs = torch.from_numpy(ref_off.view(np.int64).copy()).cuda()
    y, st, _ = gpu_dequantize(words, len(w), offs, rows, cols, p, fp32=True)
    assert st["status"] & hq.HQ_ST_CORRUPT
    ref = oracle_dequantize(ref_w, ref_off, rows, cols, O.E8, _alpha("E8"), 2, 5, 0, fp32=True)
    keep = np.ones(rows, bool)
    keep[bad] = False
    assert_recon_equal(y[keep], ref[keep])


@pytest.mark.parametrize("tokens", [1024, 3200, 4000])
def test_rotated_kv_read_every_regime(tokens):
    """8 heads: 256, 800 and 1000 chunks, around the rotation decoder's 444 / 888."""
    hq = _hq()
    H, lat, k, seed = 8, "E8", 0, 9
    L = O.LATTICES[lat]
    alpha = 0.35
    K, _ = synth.kv(H, tokens, seed=tokens)
    Q = R.haar_rotation(3)
    cache = hq.KVCache(H, tokens, hq.make_params(lat, 1.0, k, seed, 1), bits_per_scalar=16.0, max_appends=2,
                       max_append_tokens=tokens, rotation=torch.from_numpy(Q).cuda())
    cache.append(K.cuda(), alpha)
    out = torch.full((H, tokens, 128), float("nan"), device="cuda")
    cache.read(out)
    torch.cuda.synchronize()
    assert hq.read_stats(cache.stats)["status"] == 0
    s, off, _ = O.kv_append(K, 0, L, alpha, k, seed, 1, base_word=0, rot=Q)
    ref = np.zeros((H, tokens, 128), np.float32)
    O.kv_read_append(s, off, H, tokens, 0, L, alpha, k, seed, 1, ref, tokens, rot=Q)
    n = len(off) - 1
    assert np.array_equal(cache.offsets[:n + 1].cpu().numpy().view(np.uint64), off.astype(np.uint64))
    assert_recon_equal(out.cpu().numpy(), ref)


def test_gemv_two_warps_per_chunk():
    """hq_gemv at 1200 chunks (two warps per chunk without dither on a B200): the tile
    partials, then row sums, match the fp64 product of the oracle's bf16 reconstruction."""
    hq = _hq()
    rows, cols = 1200, 4096
    alpha = _alpha("E8")
    W = synth.weight(rows, cols, seed=12)
    ref_w, ref_off, _ = oracle_quantize(W, O.E8, alpha, 2, 4)
    w_bits = oracle_dequantize(ref_w, ref_off, rows, cols, O.E8, alpha, 2, 4, fp32=False)
    p = hq.make_params("E8", alpha, 2, 4, 0)
    words = torch.from_numpy(ref_w.view(np.int32).copy()).cuda()
    offs = torch.from_numpy(ref_off.view(np.int64).copy()).cuda()
    x = (torch.randn(cols, generator=torch.Generator().manual_seed(5)) * 2).to(torch.bfloat16)
    ws = torch.empty(hq.hq_gemv_workspace_bytes(rows, cols), dtype=torch.uint8, device="cuda")
    y = torch.full((rows,), float("nan"), device="cuda")
    hq.hq_gemv(words, len(ref_w), offs, rows, cols, p, x.cuda(), y, ws)
    got = y.cpu().numpy().astype(np.float64)
    w = (w_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    xv = (u16(x).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    exact, mag = w @ xv, np.abs(w) @ np.abs(xv)
    assert np.all(np.abs(got - exact) <= (40 + cols // 128) * 2.0 ** -24 * mag + 1e-30)
