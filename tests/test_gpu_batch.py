"""Strided batches (hq_quantize_batch, hq_dequantize_batch) on the GPU, through the C ABI.

One launch codes a set of equally shaped matrices; each item's stream, offsets and
stats must be exactly those of hq_quantize on that matrix alone (and so the
oracle's), and each item's reconstruction exactly hq_dequantize's.  The cases use
padded input strides, stream strides that leave items' streams unaligned, ragged
last chunks, dither, and launches large enough that warps move between items.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from hqtest import rate_points, u16

pytestmark = pytest.mark.gpu


def _hq():
    import lattice_entropy_coded_b200 as hq
    return hq


def _batch_input(B, rows, cols, seed, pad_rows=0, pad_cols=0):
    """bf16 [B, rows + pad_rows, cols + pad_cols] on the GPU; the matrices are its top-left
    [rows, cols] corners (strided views)."""
    full = torch.stack([synth.weight(rows + pad_rows, cols + pad_cols, seed=seed + i) for i in range(B)]).cuda()
    return full, full[:, :rows, :cols]


def _single(hq, x, params, cap):
    rows, cols = x.shape
    _, nch = hq.hq_stream_bound(rows, cols, params)
    words = torch.full((cap,), 7, dtype=torch.int32, device="cuda")
    offs = torch.full((nch + 1,), -1, dtype=torch.int64, device="cuda")
    st = hq.stats_tensor()
    ws = torch.empty(hq.hq_workspace_bytes(nch), dtype=torch.uint8, device="cuda")
    hq.hq_quantize(x, params, words, offs, st, ws, ld=x.stride(0))
    torch.cuda.synchronize()
    return words, offs, hq.read_stats(st)


def _batch(hq, x, params, cap, stride):
    B, rows, cols = x.shape
    _, nch = hq.hq_stream_bound(rows, cols, params)
    words = torch.full((B, stride), 7, dtype=torch.int32, device="cuda")
    offs = torch.full((B, nch + 1), -1, dtype=torch.int64, device="cuda")
    st = torch.zeros(B, hq.STATS_BYTES, dtype=torch.uint8, device="cuda")
    ws = torch.empty(hq.hq_batch_workspace_bytes(B, nch), dtype=torch.uint8, device="cuda")
    hq.hq_quantize_batch(x, params, words, offs, st, ws, cap_words=cap)
    torch.cuda.synchronize()
    return words, offs, [hq.read_stats(st[i]) for i in range(B)]


@pytest.mark.parametrize("lat,alpha,k,dither", [("E8", 314.15, 2, 0), ("E8", 175.0, 1, 0), ("D4", 183.8, 2, 1),
                                                ("Z", 160.7, 3, 0), ("A2", 123.4, 2, 0)])
@pytest.mark.parametrize("B,rows,cols", [(2, 37, 384), (5, 64, 4096), (3, 100, 1024)])
def test_batch_matches_single_calls(lat, alpha, k, dither, B, rows, cols):
    hq = _hq()
    params = hq.make_params(lat, alpha, k, 11, dither)
    full, x = _batch_input(B, rows, cols, seed=40, pad_rows=3, pad_cols=8)
    cap, _ = hq.hq_stream_bound(rows, cols, params)
    stride = cap + 13                    # items' streams start at unaligned words
    words, offs, stats = _batch(hq, x, params, cap, stride)
    out = torch.full((B, rows + 2, cols + 16), float("nan"), device="cuda")
    outb = out[:, :rows, :cols]
    st = torch.zeros(B, hq.STATS_BYTES, dtype=torch.uint8, device="cuda")
    hq.hq_dequantize_batch(words, cap, offs, rows, cols, params, outb, st)
    torch.cuda.synchronize()
    for i in range(B):
        w1, o1, s1 = _single(hq, x[i], params, cap)
        total = int(o1[-1].item())
        assert stats[i] == s1, (i, stats[i], s1)
        assert s1["status"] == 0
        assert torch.equal(offs[i], o1), i
        assert torch.equal(words[i, :total], w1[:total]), i
        assert torch.all(words[i, cap:] == 7)            # nothing written past an item's capacity
        ref = torch.empty(rows, cols, device="cuda")
        hq.hq_dequantize(w1, cap, o1, rows, cols, params, ref)
        torch.cuda.synchronize()
        assert torch.equal(outb[i], ref), i
        assert hq.read_stats(st[i])["status"] == 0
    # the padding of the output was not touched
    assert torch.isnan(out[:, rows:, :]).all() and torch.isnan(out[:, :, cols:]).all()


def test_large_batch_against_the_oracle():
    """8 matrices of 2048 x 4096 (16384 chunks in one launch, warps crossing items); items
    0 and 5 are compared word for word with the oracle, all items with single calls."""
    hq = _hq()
    B, rows, cols = 8, 2048, 4096
    params = hq.make_params("E8", 314.15, 2, 3, 0)
    full, x = _batch_input(B, rows, cols, seed=70)
    cap, _ = hq.hq_stream_bound(rows, cols, params, 64)
    words, offs, stats = _batch(hq, x, params, cap, cap)
    for i in range(B):
        w1, o1, s1 = _single(hq, x[i], params, cap)
        assert stats[i] == s1
        assert torch.equal(offs[i], o1)
        assert torch.equal(words[i, :int(o1[-1].item())], w1[:int(o1[-1].item())])
    for i in (0, 5):
        xi = x[i].cpu()
        ref_w, ref_off, ref_pb = O.quantize(u16(xi), O.E8, 314.15, 2, 3)
        got_off = offs[i].cpu().numpy().view(np.uint64)
        assert np.array_equal(got_off, ref_off)
        assert np.array_equal(words[i, :int(ref_off[-1])].cpu().numpy().view(np.uint32), ref_w)
        assert stats[i]["payload_bits"] == ref_pb
        assert (stats[i]["max_abs_code"], stats[i]["int8_overflow_count"]) == O.quantize_range(u16(xi), O.E8, 314.15, 3)


def test_batch_flags_per_item():
    """Capacity and corruption are reported on the item they concern only."""
    hq = _hq()
    B, rows, cols = 3, 64, 4096
    params = hq.make_params("E8", 314.15, 2, 5, 0)
    full, x = _batch_input(B, rows, cols, seed=90)
    x[1].mul_(64)                                        # item 1 needs a much longer stream
    cap, _ = hq.hq_stream_bound(rows, cols, params, 64)
    words, offs, stats = _batch(hq, x, params, cap, cap + 4)
    assert stats[1]["status"] & hq.HQ_ST_CAPACITY
    assert stats[1]["stream_words"] > cap
    assert stats[0]["status"] == 0 and stats[2]["status"] == 0
    assert torch.all(words[:, cap:] == 7)                # the cap held for every item
    # corrupt item 2's offsets: only its stats say so, and the other items decode
    bad = offs.clone()
    bad[2, 1], bad[2, 2] = bad[2, 2].item(), bad[2, 1].item()
    out = torch.empty(B, rows, cols, device="cuda")
    st = torch.zeros(B, hq.STATS_BYTES, dtype=torch.uint8, device="cuda")
    hq.hq_dequantize_batch(words, cap, bad, rows, cols, params, out, st)
    torch.cuda.synchronize()
    assert hq.read_stats(st[2])["status"] & hq.HQ_ST_CORRUPT
    assert hq.read_stats(st[0])["status"] == 0
    ref = torch.empty(rows, cols, device="cuda")
    w0, o0, _ = _single(hq, x[0], params, cap)
    hq.hq_dequantize(w0, cap, o0, rows, cols, params, ref)
    torch.cuda.synchronize()
    assert torch.equal(out[0], ref)


def test_student_t_set_as_benched():
    """The benchmark's launch configuration at its full size: all 64 Student-t matrices of
    8192 x 8192 (seed 4) coded by one hq_quantize_batch launch and decoded to bf16 by one
    hq_dequantize_batch launch, at each of the set's operating points (E8 3 and 4 bps).  In
    items 0, 37 and 63, sampled chunks (and each item's last) are compared word for word with
    the oracle, which computes any chunk from its row alone, and their bf16 reconstructions
    with the oracle's; every item's offsets increase and end at its stats' stream_words, with
    status 0 in both directions."""
    hq = _hq()
    B, R, Cc, seed = 64, 8192, 8192, 4
    x = torch.empty(B, R, Cc, dtype=torch.bfloat16, device="cuda")
    for i, m in enumerate(synth.student_t(B, R, Cc, seed, device="cuda")):
        x[i].copy_(m)
    out = torch.empty_like(x)
    rng = np.random.default_rng(64)
    for p in rate_points()["student_t_64x8192x8192_e8"]["points"]:
        params = hq.make_params("E8", p["alpha"], p["k"], seed, 0)
        cap = int(R * Cc * (p["bps"] + 3.0) / 32) + 8192            # the bench's capacity
        _, nch = hq.hq_stream_bound(R, Cc, params)
        words = torch.empty(B, cap, dtype=torch.int32, device="cuda")
        offs = torch.empty(B, nch + 1, dtype=torch.int64, device="cuda")
        st = torch.zeros(B, hq.STATS_BYTES, dtype=torch.uint8, device="cuda")
        dst = torch.zeros(B, hq.STATS_BYTES, dtype=torch.uint8, device="cuda")
        ws = torch.empty(hq.hq_batch_workspace_bytes(B, nch), dtype=torch.uint8, device="cuda")
        hq.hq_quantize_batch(x, params, words, offs, st, ws, cap_words=cap)
        hq.hq_dequantize_batch(words, cap, offs, R, Cc, params, out, dst)
        torch.cuda.synchronize()
        offs_c = offs.cpu().numpy().view(np.uint64)
        for i in range(B):
            s = hq.read_stats(st[i])
            assert s["status"] == 0 and hq.read_stats(dst[i])["status"] == 0, i
            assert s["stream_words"] == int(offs_c[i, -1]) <= cap
            assert offs_c[i, 0] == 0 and np.all(np.diff(offs_c[i].astype(np.int64)) > 0)
        for i in (0, 37, 63):
            wi = words[i].cpu().numpy().view(np.uint32)
            for c in [int(v) for v in rng.integers(0, nch, 3)] + [nch - 1]:
                r, h = divmod(c, 2)                  # 64 tiles per row: chunk c is half h of row r
                row = x[i, r:r + 1].cpu()
                ref_w, ref_off, _ = O.quantize(u16(row), O.E8, p["alpha"], p["k"], seed, 0, h, h + 1)
                a, b = int(offs_c[i, c]), int(offs_c[i, c + 1])
                assert np.array_equal(wi[a:b], ref_w), (p["bps"], i, c)
                ref_y = O.dequantize(ref_w, ref_off, 1, Cc, O.E8, p["alpha"], p["k"], seed, 0, False, h, h + 1)
                got = u16(out[i, r:r + 1])
                assert np.array_equal(got[0, 4096 * h:4096 * (h + 1)], ref_y[0, 4096 * h:4096 * (h + 1)]), (i, c)
        del words, offs, ws
    del x, out
    torch.cuda.empty_cache()
