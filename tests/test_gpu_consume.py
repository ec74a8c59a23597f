"""Decode fused into its consumer (hq_gemv, hq_kv_scores) against the oracle.

The matrix (or K row) a dot product sees is the oracle's bf16 reconstruction;
products of two bf16 values are exact in fp32, so the only difference from the
exact fp64 dot product is fp32 accumulation: per tile a sequential fma over a
lane's 32 elements (32 roundings), a 4-lane tree (2), then for hq_gemv the row's
tiles in column order (tiles-per-row roundings).  Each rounding contributes at
most 2^-24 of the running sum, so the error bound is
(34 + tiles_per_row) * 2^-24 * sum_j |w_j x_j|; the tests allow (40 + tpr) of it.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from hqtest import gpu_quantize, oracle_dequantize, oracle_quantize, rate_points, u16

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


def _hq():
    import lattice_entropy_coded_b200 as hq
    return hq


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _check_dot(got, w_bits, x_bits, tpr):
    w = _bf16_to_f64(w_bits)
    x = _bf16_to_f64(x_bits)
    exact = w @ x
    mag = np.abs(w) @ np.abs(x)
    lim = (40 + tpr) * U * mag + 1e-30
    err = np.abs(got.astype(np.float64) - exact)
    assert np.all(err <= lim), f"worst error / bound {float(np.max(err / lim)):.3f}"


@pytest.mark.parametrize("lat", ["E8", "D4", "A2", "Z"])
@pytest.mark.parametrize("dither", [0, 1])
@pytest.mark.parametrize("shape", [(37, 384), (64, 4096), (5, 1152), (3, 65536)])
def test_gemv_matches_the_oracle_reconstruction(lat, dither, shape):
    hq = _hq()
    rows, cols = shape
    L = O.LATTICES[lat]
    alpha = {p["lattice"]: p["alpha"] for p in rate_points()["weight_4096x4096_rate_sweep"]["points"]
             if p["bps"] == 4.0}[lat]
    W = synth.weight(rows, cols, seed=31 + rows)
    p = hq.make_params(lat, alpha, 2, 17, dither)
    g = gpu_quantize(W.cuda(), p)
    ref_w, ref_off, _ = oracle_quantize(W, L, alpha, 2, 17, dither)
    w_bits = oracle_dequantize(ref_w, ref_off, rows, cols, L, alpha, 2, 17, dither, fp32=False)
    x = (torch.randn(cols, generator=torch.Generator().manual_seed(rows)) * 3).to(torch.bfloat16)
    ws = torch.empty(hq.hq_gemv_workspace_bytes(rows, cols), dtype=torch.uint8, device="cuda")
    y = torch.full((rows,), float("nan"), device="cuda")
    st = hq.stats_tensor()
    hq.hq_gemv(g["words_t"], g["cap"], g["offsets_t"], rows, cols, p, x.cuda(), y, ws, st)
    y1 = y.cpu().numpy()
    assert hq.read_stats(st)["status"] == 0
    _check_dot(y1, w_bits, u16(x), cols // 128)
    # the same bits on every run: tile partials, then row sums in column order
    hq.hq_gemv(g["words_t"], g["cap"], g["offsets_t"], rows, cols, p, x.cuda(), y, ws, st)
    assert np.array_equal(y.cpu().numpy(), y1)


@pytest.mark.parametrize("k", [0, 8])
def test_gemv_every_remainder_path(k):
    """k = 0 (no remainder plane) and k = 8 (remainders read one by one, not in windows)."""
    hq = _hq()
    rows, cols = 21, 1024
    W = synth.weight(rows, cols, seed=77)
    alpha = 300.0 * 2 ** (k - 2) if k else 40.0
    p = hq.make_params("E8", alpha, k, 3, 0)
    g = gpu_quantize(W.cuda(), p, max_abs_symbol=1 << 14)
    ref_w, ref_off, _ = oracle_quantize(W, O.E8, alpha, k, 3)
    w_bits = oracle_dequantize(ref_w, ref_off, rows, cols, O.E8, alpha, k, 3, fp32=False)
    x = (torch.randn(cols, generator=torch.Generator().manual_seed(k)) * 2).to(torch.bfloat16)
    ws = torch.empty(hq.hq_gemv_workspace_bytes(rows, cols), dtype=torch.uint8, device="cuda")
    y = torch.empty(rows, device="cuda")
    hq.hq_gemv(g["words_t"], g["cap"], g["offsets_t"], rows, cols, p, x.cuda(), y, ws)
    _check_dot(y.cpu().numpy(), w_bits, u16(x), cols // 128)


def test_gemv_full_size_point_and_codec_method():
    """4096 x 4096 at the E8 4 bps point, through Codec.gemv, against dequantize + fp64 GEMV."""
    hq = _hq()
    pt = [q for q in rate_points()["weight_4096x4096_rate_sweep"]["points"]
          if q["lattice"] == "E8" and q["bps"] == 4.0][0]
    W = synth.weight(4096, 4096, seed=1, device="cuda")
    p = hq.make_params("E8", pt["alpha"], pt["k"], 1, 0)
    codec = hq.Codec(4096, 4096, p)
    comp = codec.quantize(W)
    wb = torch.empty(4096, 4096, dtype=torch.bfloat16, device="cuda")
    codec.dequantize(comp, wb)
    x = (torch.randn(4096, device="cuda") * 0.5).to(torch.bfloat16)
    y = torch.empty(4096, device="cuda")
    codec.gemv(comp, x, y)
    torch.cuda.synchronize()
    _check_dot(y.cpu().numpy(), u16(wb), u16(x), 32)


def test_gemv_corrupt_chunk_counts_as_zero():
    hq = _hq()
    W = synth.weight(16, 1024, seed=7)
    p = hq.make_params("E8", 300.0, 2, 1, 0)
    g = gpu_quantize(W.cuda(), p)
    off = g["offsets_t"].clone()
    off[2], off[3] = off[3], off[2]        # chunk 2 (rows 8..11) inconsistent
    x = torch.ones(1024, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(hq.hq_gemv_workspace_bytes(16, 1024), dtype=torch.uint8, device="cuda")
    y = torch.empty(16, device="cuda")
    st = hq.stats_tensor()
    hq.hq_gemv(g["words_t"], g["cap"], g["offsets_t"], 16, 1024, p, x, y, ws, st)
    good = y.cpu().numpy()
    hq.hq_gemv(g["words_t"], g["cap"], off, 16, 1024, p, x, y, ws, st)
    assert hq.read_stats(st)["status"] & hq.HQ_ST_CORRUPT
    yy = y.cpu().numpy()
    # chunk 2 is inconsistent and chunk 1 now spans chunk 2's words: both count as zero
    assert np.all(yy[4:12] == 0)
    assert np.array_equal(yy[:4], good[:4]) and np.array_equal(yy[12:], good[12:])


def _kv_ref_bits(appends, H, lat, alpha, k, seed, total):
    """The oracle's bf16 K cache, append by append."""
    ref = np.zeros((H, total, 128), np.uint16)
    t0 = 0
    for kv in appends:
        s, off, _ = O.kv_append(u16(kv), t0, lat, alpha, k, seed, 1)
        O.kv_read_append(s, off, H, kv.shape[1], t0, lat, alpha, k, seed, 1, ref, total)
        t0 += kv.shape[1]
    return ref


@pytest.mark.parametrize("lat", ["E8", "Z"])
@pytest.mark.parametrize("group", [1, 4])
def test_kv_scores_match_the_oracle_reconstruction(lat, group):
    hq = _hq()
    H, Ts = 4, [100, 1, 155]
    total = sum(Ts)
    K, _ = synth.kv(H, total, seed=8)
    L = O.LATTICES[lat]
    params = hq.make_params(lat, 1.0, 1, 23, 1)
    cache = hq.KVCache(H, total, params, bits_per_scalar=16.0, max_appends=4, max_append_tokens=256)
    appends, t0 = [], 0
    for T in Ts:
        a = K[:, t0:t0 + T].contiguous()
        appends.append(a)
        cache.append(a.cuda(), 0.4)
        t0 += T
    kbits = _kv_ref_bits(appends, H, L, 0.4, 1, 23, total)
    q = (torch.randn(H * group, 128, generator=torch.Generator().manual_seed(group)) * 0.1).to(torch.bfloat16)
    length = total - 7
    out = torch.full((H * group, total + 3), -123.0, device="cuda")
    cache.scores(q.cuda(), group, out, length)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    st = hq.read_stats(cache.stats)
    assert st["status"] == 0
    assert np.all(got[:, length:] == -123.0)            # columns >= len untouched
    qb = u16(q)
    for h in range(H):
        for gq in range(group):
            _check_dot(got[h * group + gq, :length], kbits[h, :length], qb[h * group + gq], 0)
