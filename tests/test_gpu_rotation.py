"""The dense KV rotation on the GPU against the oracle.

A KV cache may rotate each token's head vector by a full Haar-uniform 128 x 128
orthogonal matrix instead of the sign diagonal and H_128 (explainer pages,
"Methodology" 4).  The matrix is an input: the parity cases give the CUDA path and
the oracle the same fp32 matrix (the oracle's draw), and the streams, offsets and
stats must be bit-identical, the reconstructions within 1e-6 relative (they are
expected bit-identical).  The device generator is checked separately against the
oracle's draw, to within one fp32 unit in the last place.
"""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import rotation as R
import synth
from hqtest import assert_recon_equal, assert_same_words, u16

pytestmark = pytest.mark.gpu

U = 2.0**-24


def _hq():
    import lattice_entropy_coded_b200 as hq
    return hq


@pytest.mark.parametrize("seed", [0, 1, 5, 2**63 + 12345])
def test_device_haar_matches_the_oracle_draw(seed):
    hq = _hq()
    q = hq.hq_haar_rotation(seed)
    torch.cuda.synchronize()
    got = q.cpu().numpy()
    want = R.haar_rotation(seed)
    d = got.view(np.int32).astype(np.int64) - want.view(np.int32).astype(np.int64)
    assert np.abs(d).max() <= 1, f"{int((d != 0).sum())} entries differ, by up to {int(np.abs(d).max())} ulp"
    g64 = got.astype(np.float64)
    assert np.abs(g64.T @ g64 - np.eye(128)).max() < 1e-6


def _rot_cache_case(H, Ts, lat, alpha, k, seed, dither, source, Q, path=0):
    """Appends of source[:, t0:t0+T] into a rotated cache; stream, offsets, stats and the
    bf16 and fp32 reads against the oracle."""
    hq = _hq()
    Qd = torch.from_numpy(Q).cuda()
    params = hq.make_params(lat, 1.0, k, seed, dither)
    total = sum(Ts)
    cache = hq.KVCache(H, total, params, bits_per_scalar=16.0, max_appends=len(Ts) + 1,
                       max_append_tokens=max(Ts), rotation=Qd)
    hq.hq_debug_set_encode_path(path)
    try:
        t0 = 0
        appends = []
        for T in Ts:
            kv = source[:, t0:t0 + T].contiguous()
            appends.append((t0, kv))
            cache.append(kv.cuda(), alpha)
            t0 += T
    finally:
        hq.hq_debug_set_encode_path(0)
    out32 = torch.full((H, total, 128), float("nan"), device="cuda")
    out16 = torch.zeros((H, total, 128), dtype=torch.bfloat16, device="cuda")
    cache.read(out32)
    cache.read(out16)
    torch.cuda.synchronize()
    st = hq.read_stats(cache.stats)
    assert st["status"] == 0, st

    words, offs, base, pay = [], [], 0, 0
    ref32 = np.zeros((H, total, 128), np.float32)
    ref16 = np.zeros((H, total, 128), np.uint16)
    for t0, kv in appends:
        s, off, pb = O.kv_append(kv, t0, lat, alpha, k, seed, dither, base_word=base, rot=Q)
        O.kv_read_append(s, off - np.uint64(base), H, kv.shape[1], t0, lat, alpha, k, seed, dither, ref32, total,
                         rot=Q)
        O.kv_read_append(s, off - np.uint64(base), H, kv.shape[1], t0, lat, alpha, k, seed, dither, ref16, total,
                         rot=Q)
        words.append(s)
        offs.append(off[:-1])
        base = int(off[-1])
        pay += pb
    offs.append(np.array([base], np.uint64))
    ref_w, ref_off = np.concatenate(words), np.concatenate(offs)
    n = len(ref_off) - 1
    gw = cache.words[:base].cpu().numpy().view(np.uint32)
    go = cache.offsets[:n + 1].cpu().numpy().view(np.uint64)
    assert_same_words(gw, go, ref_w, ref_off)
    assert st["payload_bits"] == pay and st["stream_words"] == base
    assert_recon_equal(out32.cpu().numpy(), ref32)
    assert np.array_equal(u16(out16.cpu()), ref16)
    return cache, st


@pytest.mark.parametrize("lat", ["E8", "D4", "A2", "Z"])
@pytest.mark.parametrize("dither", [0, 1])
def test_rotated_kv_appends_and_reads_bit_exact(lat, dither):
    Q = R.haar_rotation(31)
    K, _ = synth.kv(3, 420, seed=4)
    _rot_cache_case(3, [256, 1, 31, 100, 32], O.LATTICES[lat], 0.6, 1, 19, dither, K, Q)


@pytest.mark.parametrize("k", [0, 3, 6])
@pytest.mark.parametrize("Ts", [[300], [40, 1]])
def test_rotated_kv_rice_parameters(k, Ts):
    """k <= 4 and k > 4, in the grouped form (20 chunks) and the single-CTA form (4 and 2)."""
    Q = R.haar_rotation(32)
    _, V = synth.kv(2, 300, seed=5)
    alpha = {0: 0.3, 3: 2.5, 6: 20.0}[k]
    _rot_cache_case(2, Ts, O.E8, alpha, k, 8, 1, V, Q)


def test_rotated_kv_same_stream_whatever_the_encoder_switch():
    """The rotation always runs in the grouped form: the encoder switch changes nothing."""
    Q = R.haar_rotation(33)
    K, _ = synth.kv(2, 200, seed=6)
    words = []
    for path in (0, 1, 2, 3):
        cache, _ = _rot_cache_case(2, [128, 72], O.E8, 0.5, 1, 4, 1, K, Q, path=path)
        words.append(cache.words[:int(cache.offsets[int(cache.cache.chunks)].item())].cpu().numpy())
    assert all(np.array_equal(words[0], w) for w in words[1:])


def test_rotated_kv_many_chunks():
    """8 heads x 2560 tokens: an append of 512 chunks (past one wave of 296 groups, so
    groups take several chunk tickets), then one of 128."""
    Q = R.haar_rotation(34)
    K, _ = synth.kv(8, 2560, seed=7)
    _rot_cache_case(8, [2048, 512], O.E8, 0.5, 1, 2, 1, K, Q)


def test_device_drawn_rotation_round_trips():
    """The library's own draw in a cache: with a fine lattice the read is close to the
    input (the rotation is orthogonal), and the codes differ from the default path's."""
    hq = _hq()
    Qd = hq.hq_haar_rotation(77)
    K, _ = synth.kv(2, 64, seed=9)
    params = hq.make_params("E8", 1.0, 4, 3, 1)
    rot = hq.KVCache(2, 64, params, bits_per_scalar=32.0, max_appends=2, max_append_tokens=64, rotation=Qd)
    plain = hq.KVCache(2, 64, params, bits_per_scalar=32.0, max_appends=2, max_append_tokens=64)
    kg = K.cuda()
    rot.append(kg, 8.0)
    plain.append(kg, 8.0)
    out = rot.read(torch.empty(2, 64, 128, device="cuda"))
    torch.cuda.synchronize()
    assert hq.read_stats(rot.stats)["status"] == 0
    err = (out.cpu().double() - K.double()).pow(2).sum(-1)
    assert float(err.max()) <= 16 * 4.0 / 8.0**2 * (1 + 1e-3)      # blocks * r^2 / alpha^2 (E8 with dither)
    n = int(rot.offsets[int(rot.cache.chunks)].item())
    assert not torch.equal(rot.words[:n], plain.words[:n])


def test_rotated_rate_equals_the_appends():
    hq = _hq()
    Q = R.haar_rotation(35)
    Qd = torch.from_numpy(Q).cuda()
    K, _ = synth.kv(4, 300, seed=10)
    p = hq.make_params("D4", 0.7, 1, 6, 1, rotation=Qd)
    st = hq.stats_tensor()
    hq.hq_rate_kv(K[:, 40:].contiguous().cuda(), p, st, tok0=40)
    torch.cuda.synchronize()
    got = hq.read_stats(st)
    _, off, pay = O.kv_append(K[:, 40:].contiguous(), 40, O.D4, 0.7, 1, 6, 1, rot=Q)
    assert got["payload_bits"] == pay and got["stream_words"] == int(off[-1])
    spec = hq.calib_spec(2.0, tol=0.01, k_lo=0, k_hi=2)
    res = hq.hq_calibrate_kv(K.cuda(), p, spec, st)
    assert res["k"] >= 0 and abs(res["bps"] - 2.0) <= 0.01
    _, _, pay2 = O.kv_append(K, 0, O.D4, res["alpha"], res["k"], 6, 1, rot=Q)
    assert abs(pay2 / K.numel() - res["bps"]) < 1e-12


@pytest.mark.parametrize("group", [1, 4])
def test_rotated_kv_scores(group):
    hq = _hq()
    Q = R.haar_rotation(36)
    H, Ts = 2, [100, 57]
    total = sum(Ts)
    K, _ = synth.kv(H, total, seed=11)
    params = hq.make_params("E8", 1.0, 1, 13, 1)
    cache = hq.KVCache(H, total, params, bits_per_scalar=16.0, max_appends=3, max_append_tokens=128,
                       rotation=torch.from_numpy(Q).cuda())
    ref = np.zeros((H, total, 128), np.uint16)
    t0 = 0
    for T in Ts:
        a = K[:, t0:t0 + T].contiguous()
        cache.append(a.cuda(), 0.5)
        s, off, _ = O.kv_append(a, t0, O.E8, 0.5, 1, 13, 1, rot=Q)
        O.kv_read_append(s, off, H, T, t0, O.E8, 0.5, 1, 13, 1, ref, total, rot=Q)
        t0 += T
    q = (torch.randn(H * group, 128, generator=torch.Generator().manual_seed(5)) * 0.1).to(torch.bfloat16)
    out = torch.full((H * group, total), -1.0, device="cuda")
    cache.scores(q.cuda(), group, out)
    torch.cuda.synchronize()
    assert hq.read_stats(cache.stats)["status"] == 0
    got = out.cpu().numpy().astype(np.float64)
    w = (ref.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    qb = (u16(q).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for h in range(H):
        for g in range(group):
            qh = qb[h * group + g]
            exact = w[h] @ qh
            lim = 40 * U * (np.abs(w[h]) @ np.abs(qh)) + 1e-30
            assert np.all(np.abs(got[h * group + g] - exact) <= lim)


def test_rotated_read_of_a_corrupt_chunk_is_flagged():
    """The rotated decoder on bad data: a flipped unary bit in one chunk flags HQ_ST_CORRUPT
    and zeroes that chunk's tokens; the rest of the cache reads exactly."""
    hq = _hq()
    Q = R.haar_rotation(37)
    K, _ = synth.kv(2, 96, seed=12)
    cache = hq.KVCache(2, 96, hq.make_params("E8", 1.0, 1, 5, 1), bits_per_scalar=16.0, max_appends=2,
                       max_append_tokens=96, rotation=torch.from_numpy(Q).cuda())
    cache.append(K.cuda(), 0.5)
    good = cache.read(torch.empty(2, 96, 128, device="cuda")).cpu().numpy()
    off = cache.offsets[:7].cpu().numpy().view(np.uint64)      # 2 heads x 3 chunks
    cache.words[int(off[2]) - 2] ^= 0x100                      # the last words of chunk 1 (head 0, tokens 32..63)
    bad = cache.read(torch.empty(2, 96, 128, device="cuda")).cpu().numpy()
    torch.cuda.synchronize()
    assert hq.read_stats(cache.stats)["status"] & hq.HQ_ST_CORRUPT
    assert np.all(bad[0, 32:64] == 0)
    assert np.array_equal(bad[0, :32], good[0, :32]) and np.array_equal(bad[0, 64:], good[0, 64:])
    assert np.array_equal(bad[1], good[1])
