"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Bar: lattice codes, Rice bitstreams and chunk offsets bit-identical; fp32
reconstructions within 1e-6 relative per element (they are computed with the
same fp32 operations in the same order, so they are expected bit-identical);
bf16 reconstructions bit-identical.  Inputs: the seeded synthetic workloads
(synth.py) and edge cases.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from hqtest import (POISON, assert_recon_equal, assert_same_words, gpu_dequantize, gpu_quantize, oracle_chunk,
                    oracle_dequantize, oracle_quantize, rate_points, u16)

pytestmark = pytest.mark.gpu

ALPHA_4BPS = {p["lattice"]: p["alpha"] for p in rate_points()["weight_4096x4096_rate_sweep"]["points"]
              if p["bps"] == 4.0}


def _hq():
    import lattice_entropy_coded_b200 as hq
    return hq


def _roundtrip(x_cpu, lat, alpha, k, seed, dither=0, check_bf16=True, ld=None, max_abs_symbol=0):
    hq = _hq()
    p = hq.make_params(lat, alpha, k, seed, dither)
    if ld is None:
        xg = x_cpu.cuda()
    else:
        wide = torch.zeros(x_cpu.shape[0], ld, dtype=torch.bfloat16)
        wide[:, :x_cpu.shape[1]] = x_cpu
        xg = wide.cuda()[:, :x_cpu.shape[1]]
    g = gpu_quantize(xg, p, ld=ld, max_abs_symbol=max_abs_symbol)
    ref_w, ref_off, ref_pay = oracle_quantize(x_cpu, lat, alpha, k, seed, dither)
    assert g["stats"]["status"] == 0, g["stats"]
    assert_same_words(g["words"], g["offsets"], ref_w, ref_off)
    assert g["stats"]["payload_bits"] == ref_pay
    assert g["stats"]["stream_words"] == len(ref_w)
    rows, cols = x_cpu.shape
    y, st, _ = gpu_dequantize(g["words_t"], g["cap"], g["offsets_t"], rows, cols, p, fp32=True)
    assert st["status"] == 0
    ref_y = oracle_dequantize(ref_w, ref_off, rows, cols, lat, alpha, k, seed, dither, fp32=True)
    assert_recon_equal(y, ref_y)
    if check_bf16:
        yb, st, _ = gpu_dequantize(g["words_t"], g["cap"], g["offsets_t"], rows, cols, p, fp32=False)
        ref_b = oracle_dequantize(ref_w, ref_off, rows, cols, lat, alpha, k, seed, dither, fp32=False)
        assert np.array_equal(yb, ref_b)
    return g, y


@pytest.mark.parametrize("lat", ["E8", "D4", "A2", "Z"])
@pytest.mark.parametrize("dither", [0, 1])
@pytest.mark.parametrize("shape", [(37, 384), (1, 128), (64, 4096), (5, 1152)])
def test_weights_bit_exact_small(lat, dither, shape):
    """Several chunks and a ragged last chunk (37x384 = 111 tiles = 3 full chunks + 15 tiles)."""
    x = synth.weight(*shape, seed=11 + shape[0])
    _roundtrip(x, O.LATTICES[lat], ALPHA_4BPS[lat], 2, seed=1234 + shape[1], dither=dither)


@pytest.mark.parametrize("k", [0, 1, 3, 4, 5, 8, 11, 15])
def test_every_rice_parameter(k):
    x = synth.weight(40, 512, seed=3)
    _roundtrip(x, O.E8, 300.0 * 2 ** (k - 2) if k < 8 else 300.0, k, seed=7)


@pytest.mark.parametrize("k", [1, 2, 3, 4])
@pytest.mark.parametrize("dither", [0, 1])
def test_rice_parameter_compiled_in(k, dither):
    """E8 weights at k = 1 .. 4 with rows that hold whole rounds (cols a multiple of 1024), forced
    onto the per-warp form: the bulk-input encoder and the bf16 decoder instantiations with k
    compiled in (with and without dither), and at k = 0 the runtime-k ones, against the oracle."""
    hq = _hq()
    hq.hq_debug_set_encode_path(1)
    try:
        x = synth.weight(40, 2048, seed=11)
        _roundtrip(x, O.E8, 300.0 * 2 ** (k - 2), k, seed=7, dither=dither)
        if k == 1:
            _roundtrip(x, O.E8, 40.0, 0, seed=7, dither=dither)
    finally:
        hq.hq_debug_set_encode_path(0)


def test_strided_rows():
    x = synth.weight(33, 256, seed=4)
    _roundtrip(x, O.E8, 300.0, 2, seed=5, ld=512)


def test_all_zero_and_tiny_alpha():
    x = torch.zeros(16, 256, dtype=torch.bfloat16)
    g, y = _roundtrip(x, O.E8, 300.0, 2, seed=1)
    assert np.all(y == 0)
    x = synth.weight(16, 256, seed=9)
    _roundtrip(x, O.E8, 1e-3, 0, seed=1)   # every code is the origin


def test_ties_and_structured_inputs():
    """Constant tiles, exact powers of two and +-0: many exact ties in rounding and in the argmax."""
    x = torch.zeros(32, 256)
    x[0] = 1.0
    x[1] = -1.0
    x[2, ::2] = 0.5
    x[3] = torch.arange(256) % 7 - 3.0
    x[4] = -0.0
    x[5, :128] = 2.0 ** -130      # bf16 subnormal
    x[6] = torch.linspace(-4, 4, 256)
    x = x.to(torch.bfloat16)
    for lat in ("E8", "D4", "A2", "Z"):
        for alpha in (1.0, 11.3137085, 64.0):    # 11.31 ~ sqrt(128): scaled values land on ties
            _roundtrip(x, O.LATTICES[lat], alpha, 1, seed=3)


def test_large_symbols_take_the_slow_path_with_the_same_bits():
    """alpha so large that chunks exceed the shared stage and quotients exceed 255."""
    x = synth.weight(64, 512, seed=12)
    g, _ = _roundtrip(x, O.E8, 40000.0, 2, seed=2, max_abs_symbol=1 << 14)
    assert g["total"] / len(g["offsets"]) > 2048       # > stage size per chunk
    assert g["stats"]["max_symbol"] >> 10                # quotients above 255
    g, _ = _roundtrip(x, O.Z, 3000.0, 0, seed=2, max_abs_symbol=1 << 14)


def test_config1_weight_tile_full():
    p = rate_points()["weight_1024x1024_e8_4bps"]["points"][0]
    x = synth.weight(1024, 1024, seed=0)
    g, y = _roundtrip(x, O.E8, p["alpha"], p["k"], seed=0)
    bps = g["stats"]["payload_bits"] / x.numel()
    assert abs(bps - 4.0) < 0.01


def test_config2_rate_sweep_full():
    """4096x4096, all 12 (lattice, rate) points at full size."""
    x = synth.weight(4096, 4096, seed=1)
    xg = x.cuda()
    hq = _hq()
    for p in rate_points()["weight_4096x4096_rate_sweep"]["points"]:
        lat = O.LATTICES[p["lattice"]]
        params = hq.make_params(lat, p["alpha"], p["k"], 1, 0)
        g = gpu_quantize(xg, params)
        ref_w, ref_off, ref_pay = oracle_quantize(x, lat, p["alpha"], p["k"], 1)
        assert g["stats"]["status"] == 0
        assert_same_words(g["words"], g["offsets"], ref_w, ref_off)
        assert abs(g["stats"]["payload_bits"] / x.numel() - p["bps"]) < 0.01
        y, st, _ = gpu_dequantize(g["words_t"], g["cap"], g["offsets_t"], 4096, 4096, params, fp32=True)
        ref_y = oracle_dequantize(ref_w, ref_off, 4096, 4096, lat, p["alpha"], p["k"], 1, 0, fp32=True)
        assert_recon_equal(y, ref_y)


# ------------------------------------------------------------------ KV cache
def _kv_oracle(appends, H, lat, alphas, k, seed, dither=1):
    """Oracle stream of a cache built from `appends` (list of [H, T, 128] bf16)."""
    words, offs, base, tok0, tables = [], [], 0, 0, []
    for kv, a in zip(appends, alphas):
        s, off, _ = O.kv_append(kv, tok0, lat, a, k, seed, dither, base_word=base)
        words.append(s)
        offs.append(off[:-1])
        tables.append((tok0, kv.shape[1], a, off))
        base = int(off[-1])
        tok0 += kv.shape[1]
    offs.append(np.array([base], np.uint64))
    return np.concatenate(words), np.concatenate(offs), tables


def _kv_case(H, Ts, lat, alpha, k, seed, dither, source):
    hq = _hq()
    params = hq.make_params(lat, 1.0, k, seed, dither)
    total_t = sum(Ts)
    cache = hq.KVCache(H, total_t, params, bits_per_scalar=16.0, max_appends=len(Ts) + 1,
                       max_append_tokens=max(Ts))
    appends, t0 = [], 0
    for T in Ts:
        kv = source[:, t0:t0 + T].contiguous()
        t0 += T
        appends.append(kv)
        cache.append(kv.cuda(), alpha)
    out = torch.full((H, total_t, 128), float("nan"), device="cuda")
    cache.read(out)
    torch.cuda.synchronize()
    st = hq.read_stats(cache.stats)
    assert st["status"] == 0, st
    ref_w, ref_off, tables = _kv_oracle(appends, H, lat, [alpha] * len(Ts), k, seed, dither)
    n = len(ref_off) - 1
    gw = cache.words[:int(ref_off[-1])].cpu().numpy().view(np.uint32)
    go = cache.offsets[:n + 1].cpu().numpy().view(np.uint64)
    assert_same_words(gw, go, ref_w, ref_off)
    ref_y = np.zeros((H, total_t, 128), np.float32)
    for (tok0, T, a, off) in tables:
        O.kv_read_append(ref_w, off, H, T, tok0, lat, a, k, seed, dither, ref_y, total_t)
    assert_recon_equal(out.cpu().numpy(), ref_y)
    return cache


@pytest.mark.parametrize("lat", ["E8", "D4", "A2", "Z"])
def test_kv_appends_bit_exact(lat):
    K, V = synth.kv(4, 700, seed=2)
    _kv_case(4, [256, 100, 1, 31, 312], O.LATTICES[lat], 0.5, 1, seed=77, dither=1, source=K)


def test_kv_appends_k0_bit_exact():
    """E8 with dither at k = 0 (the caches' rates near 2 bits): the KV-only encoder and the bf16
    read decoder with k compiled in, and a prefill-sized append (one launch of 2048 tokens)."""
    K, _ = synth.kv(4, 2700, seed=3)
    cache = _kv_case(4, [256, 100, 1, 31, 312, 2000], O.E8, 0.17, 0, seed=78, dither=1, source=K)
    # the bf16 read is the round-to-nearest-even of the fp32 read (checked against the oracle above)
    y32 = torch.empty(4, 2700, 128, device="cuda")
    y16 = torch.empty(4, 2700, 128, dtype=torch.bfloat16, device="cuda")
    cache.read(y32)
    cache.read(y16)
    torch.cuda.synchronize()
    assert torch.equal(y16, y32.to(torch.bfloat16))


def test_kv_config3_full_size():
    """8 heads x 32768 tokens, appends of 256 tokens, E8 with dither at the calibrated 2.0 bps point."""
    K, V = synth.kv(8, 32768, seed=2)
    pts = {(p["tensor"], p["bps"]): p for p in rate_points()["kv_8h_32768tok_e8_dither"]["points"]}
    for name, src in (("K", K), ("V", V)):
        p = pts[(name, 2.0)]
        cache = _kv_case(8, [256] * 128, O.E8, p["alpha"], p["k"], seed=2, dither=1, source=src)
        hq = _hq()
        bps = hq.read_stats(cache.stats)["payload_bits"] / src.numel()
        assert abs(bps - 2.0) < 0.02


def test_kv_read_prefix_length():
    hq = _hq()
    K, _ = synth.kv(2, 300, seed=5)
    params = hq.make_params("E8", 1.0, 0, 9, 1)
    cache = hq.KVCache(2, 300, params, max_appends=4, max_append_tokens=256)
    cache.append(K[:, :256].contiguous().cuda(), 0.2)
    cache.append(K[:, 256:].contiguous().cuda(), 0.3)
    full = torch.zeros(2, 300, 128, device="cuda")
    cache.read(full)
    part = torch.full((2, 300, 128), 7.0, device="cuda")
    cache.read(part, 270)
    torch.cuda.synchronize()
    assert torch.equal(part[:, :270], full[:, :270])
    assert torch.all(part[:, 270:] == 7.0)


# ------------------------------------------------------------------ full-size workloads, sampled
def _sampled_check(x_gpu, params, lat, alpha, k, seed, n_samples=24, rng=None):
    g = gpu_quantize(x_gpu, params, cap_words=int(x_gpu.numel() * 6 // 32) + 4096)
    assert g["stats"]["status"] == 0
    rows, cols = x_gpu.shape
    nch = len(g["offsets"]) - 1
    rng = rng or np.random.default_rng(0)
    picks = sorted(set([0, nch - 1] + list(rng.integers(0, nch, n_samples))))
    tpr = cols // 128
    for c in picks:
        r0, r1 = (32 * c) // tpr, min(rows, (32 * c + 31) // tpr + 1)
        sub = x_gpu[r0:r1].cpu()
        # chunk c's tiles, re-indexed into the row slice (tile 32c is at row r0)
        lc = (32 * c - r0 * tpr) // 32
        assert (32 * c - r0 * tpr) % 32 == 0 or tpr % 32 == 0
        w_ref, _ = oracle_chunk(sub, lc, lat, alpha, k, seed)
        a, b = int(g["offsets"][c]), int(g["offsets"][c + 1])
        assert np.array_equal(g["words"][a:b], w_ref), f"chunk {c}"
    return g


def test_weight_set_8b_full_size_sampled():
    hq = _hq()
    p = rate_points()["weights_8b_8layers_e8_4bps"]["points"][0]
    rng = np.random.default_rng(3)
    for i, (name, w) in enumerate(synth.weight_set(3, device="cuda")):
        if i % 9 and i != 55:            # every shape, in several layers, and the last matrix
            continue
        params = hq.make_params("E8", p["alpha"], p["k"], 3, 0)
        _sampled_check(w, params, O.E8, p["alpha"], p["k"], 3, n_samples=6, rng=rng)


def test_student_t_full_size_sampled():
    hq = _hq()
    rng = np.random.default_rng(4)
    pts = rate_points()["student_t_64x8192x8192_e8"]["points"]
    for i, m in enumerate(synth.student_t(3, 8192, 8192, 4, device="cuda")):
        p = pts[i % 2]
        params = hq.make_params("E8", p["alpha"], p["k"], 4, 0)
        g = _sampled_check(m, params, O.E8, p["alpha"], p["k"], 4, n_samples=8, rng=rng)
        # decode sampled rows
        y, st, _ = gpu_dequantize(g["words_t"], g["cap"], g["offsets_t"], 8192, 8192, params, fp32=True)
        assert st["status"] == 0
        for c in rng.integers(0, len(g["offsets"]) - 1, 3):
            a, b = int(g["offsets"][c]), int(g["offsets"][c + 1])
            q = O.decode_chunk(O.E8, p["k"], g["words"][a:b], 32)
            r = (32 * int(c)) // 64
            tc0 = (32 * int(c)) % 64
            for t in range(32):
                ref = O.dequantize_tile(q[t * 128:(t + 1) * 128], O.E8, p["alpha"], 4, (tc0 + t) * 128)
                got = y[r, (tc0 + t) * 128:(tc0 + t + 1) * 128]
                assert_recon_equal(got, ref)


# ------------------------------------------------------------------ faults (made on the host)
def test_capacity_overflow_is_flagged_and_bounded():
    hq = _hq()
    x = synth.weight(64, 1024, seed=6).cuda()
    params = hq.make_params("E8", 300.0, 2, 1, 0)
    full = gpu_quantize(x, params)
    need = full["total"]
    cap = need // 2
    g = gpu_quantize(x, params, cap_words=cap, guard=256)
    assert g["stats"]["status"] & hq.HQ_ST_CAPACITY
    assert g["stats"]["stream_words"] == need
    assert np.array_equal(g["offsets"], full["offsets"])
    assert np.array_equal(g["all_words"][:cap], full["words"][:cap])
    assert np.all(g["all_words"][cap:] == np.uint32(POISON))   # nothing written past the cap


def test_corrupt_streams_are_flagged():
    hq = _hq()
    x = synth.weight(16, 1024, seed=7)
    params = hq.make_params("E8", 300.0, 2, 1, 0)
    g = gpu_quantize(x.cuda(), params)
    # (a) offsets not monotone
    off = g["offsets_t"].clone()
    off[2], off[3] = off[3], off[2]
    y, st, _ = gpu_dequantize(g["words_t"], g["cap"], off, 16, 1024, params)
    assert st["status"] & hq.HQ_ST_CORRUPT
    assert np.all(y[2 * 4:3 * 4] == 0)             # chunk 2 (rows 8..11) zeroed
    # (b) offsets beyond the stream
    y, st, _ = gpu_dequantize(g["words_t"], g["total"] - 5, g["offsets_t"], 16, 1024, params)
    assert st["status"] & hq.HQ_ST_CORRUPT
    # (c) a flipped bit in a unary plane changes the terminator count
    w = g["words_t"].clone()
    a, b = int(g["offsets"][1]), int(g["offsets"][2])
    w[b - 3] ^= 0x10
    y, st, _ = gpu_dequantize(w, g["cap"], g["offsets_t"], 16, 1024, params)
    assert st["status"] & hq.HQ_ST_CORRUPT
    # the other chunks still decode exactly
    good, _, _ = gpu_dequantize(g["words_t"], g["cap"], g["offsets_t"], 16, 1024, params)
    assert np.array_equal(y[:4], good[:4]) and np.array_equal(y[8:], good[8:])


def test_lookback_spin_limit_never_hangs():
    """With a one-poll look-back limit a chunk whose predecessor is late gives up and
    flags HQ_ST_TIMEOUT; the call returns, writes stay in bounds, and if no chunk
    timed out the stream is exact."""
    hq = _hq()
    x = synth.weight(2048, 4096, seed=8).cuda()
    params = hq.make_params("E8", 300.0, 2, 1, 0)
    ref = gpu_quantize(x, params)
    hq.hq_debug_set_spin_limit(1)
    try:
        g = gpu_quantize(x, params, guard=64)
    finally:
        hq.hq_debug_set_spin_limit(0)
    assert g["stats"]["status"] & ~hq.HQ_ST_TIMEOUT == 0 or g["stats"]["status"] & hq.HQ_ST_CAPACITY
    assert np.all(g["all_words"][g["cap"]:] == np.uint32(POISON))
    if not g["stats"]["status"] & hq.HQ_ST_TIMEOUT:
        assert np.array_equal(g["words"], ref["words"])
    again = gpu_quantize(x, params)
    assert np.array_equal(again["words"], ref["words"])


def test_empty_matrix():
    hq = _hq()
    params = hq.make_params("E8", 300.0, 2, 1, 0)
    x = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    g = gpu_quantize(x, params)
    assert g["total"] == 0 and g["stats"]["status"] == 0
