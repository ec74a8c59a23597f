"""The second Rice parameter on the GPU against the oracle.

Bit-stripping halves the last symbol of each A2, D4 and E8 block; with
`rice_dk_last` > 0 that symbol is coded with max(k - dk_last, 0).  Every encoder form,
the decoder, the fused consumers, the KV path (with and without the dense rotation),
the rate pass and calibration take the mode; streams, offsets and stats must be
bit-identical to the oracle's, reconstructions equal to it.
"""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import rotation as R
import synth
from hqtest import (assert_recon_equal, assert_same_words, gpu_dequantize, gpu_quantize, oracle_dequantize,
                    oracle_quantize, u16)

pytestmark = pytest.mark.gpu

ALPHA = {"E8": 314.15, "D4": 183.8, "A2": 130.0, "Z": 90.0}


def _hq():
    import lattice_entropy_coded_b200 as hq
    return hq


def _roundtrip(x, lat, alpha, k, dk, seed=3, dither=0, path=0, max_abs_symbol=0):
    hq = _hq()
    L = O.LATTICES[lat]
    p = hq.make_params(lat, alpha, k, seed, dither, dk_last=dk)
    hq.hq_debug_set_encode_path(path)
    try:
        g = gpu_quantize(x.cuda(), p, max_abs_symbol=max_abs_symbol)
    finally:
        hq.hq_debug_set_encode_path(0)
    ref_w, ref_off, ref_pay = oracle_quantize(x, L, alpha, k, seed, dither, dk_last=dk)
    assert g["stats"]["status"] == 0, g["stats"]
    assert_same_words(g["words"], g["offsets"], ref_w, ref_off)
    assert g["stats"]["payload_bits"] == ref_pay and g["stats"]["stream_words"] == len(ref_w)
    rows, cols = x.shape
    y, st, _ = gpu_dequantize(g["words_t"], g["cap"], g["offsets_t"], rows, cols, p, fp32=True)
    assert st["status"] == 0
    assert_recon_equal(y, oracle_dequantize(ref_w, ref_off, rows, cols, L, alpha, k, seed, dither, fp32=True,
                                            dk_last=dk))
    yb, _, _ = gpu_dequantize(g["words_t"], g["cap"], g["offsets_t"], rows, cols, p, fp32=False)
    assert np.array_equal(yb, oracle_dequantize(ref_w, ref_off, rows, cols, L, alpha, k, seed, dither, fp32=False,
                                                dk_last=dk))
    st = hq.stats_tensor()
    hq.hq_rate(x.cuda(), p, st)
    torch.cuda.synchronize()
    r = hq.read_stats(st)
    assert r["payload_bits"] == ref_pay and r["stream_words"] == len(ref_w)
    return g, ref_pay


@pytest.mark.parametrize("path", [0, 1, 2, 3])
@pytest.mark.parametrize("lat", ["E8", "D4", "A2", "Z"])
@pytest.mark.parametrize("dither", [0, 1])
def test_two_k_weights_every_form(path, lat, dither):
    """Every encoder form (3, the wide one, falls back to the grouped form in this mode)
    on several chunks and a ragged last one."""
    x = synth.weight(37, 384, seed=21)
    _roundtrip(x, lat, ALPHA[lat], 2, 1, dither=dither, path=path)


@pytest.mark.parametrize("k,dk", [(0, 1), (1, 1), (2, 2), (3, 1), (4, 3), (5, 1), (8, 2), (15, 4), (2, 9)])
def test_two_k_rice_parameters(k, dk):
    """k <= 4 and k > 4 (group windows of up to 32 bits, and per-symbol reads), dk larger
    than k (the last symbol at k = 0)."""
    for lat in ("E8", "A2"):
        x = synth.weight(24, 512, seed=22 + k)
        alpha = ALPHA[lat] * 2.0 ** (k - 2) if k <= 8 else ALPHA[lat] * 8
        _roundtrip(x, lat, alpha, k, dk, path=1)
        _roundtrip(x, lat, alpha, k, dk, path=2)


def test_two_k_saves_bits_at_4_bps():
    x = synth.weight(256, 4096, seed=1)
    for lat, dk in (("E8", 1), ("D4", 1), ("A2", 2)):
        _, p0 = _roundtrip(x, lat, ALPHA[lat], 2 if lat != "A2" else 3, 0, path=1)
        _, p1 = _roundtrip(x, lat, ALPHA[lat], 2 if lat != "A2" else 3, dk, path=1)
        assert p1 < p0


def test_two_k_large_symbols_slow_path():
    """Chunks beyond the shared stage are set bit by bit in global memory, in this mode too."""
    x = synth.weight(64, 512, seed=12)
    for path in (1, 2):
        g, _ = _roundtrip(x, "E8", 40000.0, 2, 1, path=path, max_abs_symbol=1 << 14)
        assert g["total"] / len(g["offsets"]) > 1024


@pytest.mark.parametrize("rot", [False, True])
@pytest.mark.parametrize("H", [3, 8])
def test_two_k_kv_cache(rot, H):
    """3 heads: every append fits the single-CTA form; 8 heads: the 100- and 155-token
    appends (32 and 40 chunks) take the multi-CTA forms."""
    hq = _hq()
    Ts = [100, 1, 155]
    total = sum(Ts)
    K, _ = synth.kv(H, total, seed=23)
    Q = R.haar_rotation(41) if rot else None
    params = hq.make_params("D4", 1.0, 2, 5, 1, dk_last=1)
    cache = hq.KVCache(H, total, params, bits_per_scalar=16.0, max_appends=4, max_append_tokens=256,
                       rotation=torch.from_numpy(Q).cuda() if rot else None)
    words, offs, base, t0 = [], [], 0, 0
    ref = np.zeros((H, total, 128), np.float32)
    for T in Ts:
        a = K[:, t0:t0 + T].contiguous()
        cache.append(a.cuda(), 1.3)
        s, off, _ = O.kv_append(a, t0, O.D4, 1.3, 2, 5, 1, base_word=base, rot=Q, dk_last=1)
        O.kv_read_append(s, off - np.uint64(base), H, T, t0, O.D4, 1.3, 2, 5, 1, ref, total, rot=Q, dk_last=1)
        words.append(s)
        offs.append(off[:-1])
        base = int(off[-1])
        t0 += T
    offs.append(np.array([base], np.uint64))
    out = torch.full((H, total, 128), float("nan"), device="cuda")
    cache.read(out)
    torch.cuda.synchronize()
    assert hq.read_stats(cache.stats)["status"] == 0
    n = len(np.concatenate(offs)) - 1
    assert_same_words(cache.words[:base].cpu().numpy().view(np.uint32), cache.offsets[:n + 1].cpu().numpy().view(np.uint64),
                      np.concatenate(words), np.concatenate(offs))
    assert_recon_equal(out.cpu().numpy(), ref)
    # scores straight from the cache: the same bf16 rows as the read
    q = (torch.randn(H, 128, generator=torch.Generator().manual_seed(2)) * 0.1).to(torch.bfloat16)
    sc = cache.scores(q.cuda(), 1, torch.empty(H, total, device="cuda"))
    kb = torch.from_numpy(ref).to(torch.bfloat16).double()
    want = torch.einsum("htd,hd->ht", kb, q.double())
    mag = torch.einsum("htd,hd->ht", kb.abs(), q.double().abs())
    assert bool(((sc.cpu().double() - want).abs() <= 40 * 2.0**-24 * mag + 1e-30).all())


def test_two_k_gemv():
    hq = _hq()
    W = synth.weight(48, 1024, seed=24)
    p = hq.make_params("A2", ALPHA["A2"], 3, 2, 0, dk_last=2)
    g = gpu_quantize(W.cuda(), p)
    ref_w, ref_off, _ = oracle_quantize(W, O.A2, ALPHA["A2"], 3, 2, dk_last=2)
    assert_same_words(g["words"], g["offsets"], ref_w, ref_off)
    wb = oracle_dequantize(ref_w, ref_off, 48, 1024, O.A2, ALPHA["A2"], 3, 2, fp32=False, dk_last=2)
    x = (torch.randn(1024, generator=torch.Generator().manual_seed(4)) * 0.5).to(torch.bfloat16)
    ws = torch.empty(hq.hq_gemv_workspace_bytes(48, 1024), dtype=torch.uint8, device="cuda")
    y = torch.empty(48, device="cuda")
    hq.hq_gemv(g["words_t"], g["cap"], g["offsets_t"], 48, 1024, p, x.cuda(), y, ws)
    torch.cuda.synchronize()
    w = (wb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    xv = (u16(x).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    lim = (40 + 8) * 2.0**-24 * (np.abs(w) @ np.abs(xv)) + 1e-30
    assert np.all(np.abs(y.cpu().numpy().astype(np.float64) - w @ xv) <= lim)


def test_two_k_calibration():
    """Calibration in this mode: the rate it lands on is the oracle's at its alpha and k."""
    hq = _hq()
    x = synth.weight(512, 1024, seed=25)
    p = hq.make_params("E8", 1.0, 0, 9, 0, dk_last=1)
    res = hq.hq_calibrate(x.cuda(), p, hq.calib_spec(4.0, tol=0.002, k_lo=1, k_hi=4), hq.stats_tensor())
    assert res["k"] >= 1 and abs(res["bps"] - 4.0) <= 0.002
    _, _, pay = oracle_quantize(x, O.E8, res["alpha"], res["k"], 9, dk_last=1)
    assert pay / x.numel() == res["bps"]


def test_two_k_static_entry_point():
    """hq_quantize_static (no workspace) gives hq_quantize's stream in this mode too, in the
    single-CTA form (16 chunks) and in the multi-CTA forms (64 chunks)."""
    hq = _hq()
    for rows in (64, 256):
        x = synth.weight(rows, 1024, seed=26).cuda()
        p = hq.make_params("A2", ALPHA["A2"], 3, 4, 0, dk_last=2)
        ref = gpu_quantize(x, p)
        bound, nch = hq.hq_stream_bound(rows, 1024, p)
        words = torch.empty(bound, dtype=torch.int32, device="cuda")
        offs = torch.empty(nch + 1, dtype=torch.int64, device="cuda")
        st = hq.stats_tensor()
        hq.hq_quantize_static(x, p, words, offs, st)
        torch.cuda.synchronize()
        assert hq.read_stats(st) == ref["stats"]
        assert np.array_equal(offs.cpu().numpy().view(np.uint64), ref["offsets"])
        assert np.array_equal(words[:ref["total"]].cpu().numpy().view(np.uint32), ref["words"])


def test_two_k_corrupt_streams_are_flagged():
    """The decoder's MIXED variant on bad data: swapped offsets and a flipped unary bit
    flag HQ_ST_CORRUPT and zero that chunk's tiles; the other chunks decode exactly."""
    hq = _hq()
    x = synth.weight(16, 1024, seed=27)
    p = hq.make_params("D4", ALPHA["D4"], 2, 3, 0, dk_last=1)
    g = gpu_quantize(x.cuda(), p)
    good, st, _ = gpu_dequantize(g["words_t"], g["cap"], g["offsets_t"], 16, 1024, p)
    assert st["status"] == 0
    off = g["offsets_t"].clone()
    off[2], off[3] = off[3], off[2]
    y, st, _ = gpu_dequantize(g["words_t"], g["cap"], off, 16, 1024, p)
    assert st["status"] & hq.HQ_ST_CORRUPT
    assert np.all(y[8:12] == 0)
    assert np.array_equal(y[:4], good[:4]) and np.array_equal(y[12:], good[12:])
    w = g["words_t"].clone()
    b = int(g["offsets"][2])
    w[b - 3] ^= 0x10
    y, st, _ = gpu_dequantize(w, g["cap"], g["offsets_t"], 16, 1024, p)
    assert st["status"] & hq.HQ_ST_CORRUPT
    assert np.array_equal(y[:4], good[:4]) and np.array_equal(y[8:], good[8:])
