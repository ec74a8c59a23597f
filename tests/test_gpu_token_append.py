"""One-token KV appends (every chunk one tile) against the oracle, with and without the
dense rotation.

A decode step appends one token per head.  The single-CTA encoder then gives each
chunk to a half-warp in the wide layout (16 lanes to the tile), so these cases run a
code path of their own: every lattice, with and without dither, Rice parameters on
both sides of the packed-remainder limit, 1 to 32 heads, one-token appends between
longer ones, and tiles whose codes do not fit the path's stage."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
import test_gpu_parity as P
from hqtest import assert_recon_equal, assert_same_words

pytestmark = pytest.mark.gpu


def _hq():
    import lattice_entropy_coded_b200 as hq
    return hq


def _case(H, Ts, lat, alpha, k, seed, dither, source, bits_per_scalar=16.0):
    hq = _hq()
    L = O.LATTICES[lat]
    params = hq.make_params(lat, 1.0, k, seed, dither)
    total = sum(Ts)
    cache = hq.KVCache(H, total, params, bits_per_scalar=bits_per_scalar, max_appends=len(Ts) + 1,
                       max_append_tokens=max(Ts))
    appends, t0 = [], 0
    for T in Ts:
        kv = source[:, t0:t0 + T].contiguous()
        t0 += T
        appends.append(kv)
        cache.append(kv.cuda(), alpha)
    out = torch.full((H, total, 128), float("nan"), device="cuda")
    cache.read(out)
    torch.cuda.synchronize()
    st = hq.read_stats(cache.stats)
    assert st["status"] == 0, st
    ref_w, ref_off, tables = P._kv_oracle(appends, H, L, [alpha] * len(Ts), k, seed, dither)
    n = len(ref_off) - 1
    assert_same_words(cache.words[:int(ref_off[-1])].cpu().numpy().view(np.uint32),
                      cache.offsets[:n + 1].cpu().numpy().view(np.uint64), ref_w, ref_off)
    ref_y = np.zeros((H, total, 128), np.float32)
    for (tok0, T, a, off) in tables:
        O.kv_read_append(ref_w, off, H, T, tok0, L, a, k, seed, dither, ref_y, total)
    assert_recon_equal(out.cpu().numpy(), ref_y)
    return st


ALPHA = {"E8": 0.35, "D4": 0.3, "A2": 0.25, "Z": 0.3}   # about 2 bps at k = 0 on N(0, 1)


@pytest.mark.parametrize("lat", ["E8", "D4", "A2", "Z"])
@pytest.mark.parametrize("dither", [0, 1])
@pytest.mark.parametrize("k", [0, 2, 6])
def test_one_token_appends(lat, dither, k):
    K, V = synth.kv(8, 40, seed=k + 3)
    _case(8, [1] * 12 + [17] + [1] * 5, lat, ALPHA[lat] * 2.0 ** k, k, seed=11 + k, dither=dither,
          source=V if dither else K)


@pytest.mark.parametrize("H", [1, 2, 31, 32])
def test_head_counts(H):
    """1 to 32 heads (32 one-tile chunks is the single-CTA limit; 33 would take the other forms)."""
    K, _ = synth.kv(H, 9, seed=H)
    _case(H, [1] * 9, "E8", 0.7, 1, seed=5, dither=1, source=K)


def test_thirty_three_heads_take_another_form():
    K, _ = synth.kv(33, 4, seed=33)
    _case(33, [1] * 4, "E8", 0.7, 1, seed=5, dither=1, source=K)


@pytest.mark.parametrize("dither", [0, 1])
def test_tile_larger_than_the_stage(dither):
    """k = 0 and a large alpha: quotients in the hundreds, so a tile's unary plane runs past
    the path's 256-word stage and the chunk is set in place in global memory instead."""
    K, _ = synth.kv(4, 3, seed=8)
    st = _case(4, [1, 1, 1], "E8", 40.0, 0, seed=3, dither=dither, source=K, bits_per_scalar=512.0)
    assert st["payload_bits"] > 4 * 3 * 256 * 32   # the stage's bound, exceeded on average


def test_forms_agree_on_one_token():
    """The same one-token appends through each forced encoder form give one stream."""
    hq = _hq()
    K, _ = synth.kv(8, 6, seed=21)
    outs = []
    for path in (1, 2, 3, 4):
        hq.hq_debug_set_encode_path(path)
        try:
            params = hq.make_params("D4", 1.0, 2, 9, 1)
            cache = hq.KVCache(8, 6, params, bits_per_scalar=16.0, max_appends=7, max_append_tokens=1)
            for t in range(6):
                cache.append(K[:, t:t + 1].contiguous().cuda(), 1.2)
            torch.cuda.synchronize()
            n = 8 * 6
            end = int(cache.offsets[n].item())
            outs.append((cache.words[:end].cpu().numpy().copy(), cache.offsets[:n + 1].cpu().numpy().copy()))
        finally:
            hq.hq_debug_set_encode_path(0)
    for w, o in outs[1:]:
        assert np.array_equal(o, outs[0][1]) and np.array_equal(w, outs[0][0])


def _rot_case(H, Ts, lat, alpha, k, seed, dither, source, rot_seed):
    """The same with a dense Haar rotation per cache, against the oracle's rotated path."""
    from oracle import rotation as R
    hq = _hq()
    L = O.LATTICES[lat]
    Q = R.haar_rotation(rot_seed)
    total = sum(Ts)
    cache = hq.KVCache(H, total, hq.make_params(lat, 1.0, k, seed, dither), bits_per_scalar=16.0,
                       max_appends=len(Ts) + 1, max_append_tokens=max(Ts), rotation=torch.from_numpy(Q).cuda())
    words, offs, base, t0 = [], [], 0, 0
    ref = np.zeros((H, total, 128), np.float32)
    for T in Ts:
        a = source[:, t0:t0 + T].contiguous()
        cache.append(a.cuda(), alpha)
        s, off, _ = O.kv_append(a, t0, L, alpha, k, seed, dither, base_word=base, rot=Q)
        O.kv_read_append(s, off - np.uint64(base), H, T, t0, L, alpha, k, seed, dither, ref, total, rot=Q)
        words.append(s)
        offs.append(off[:-1])
        base = int(off[-1])
        t0 += T
    offs.append(np.array([base], np.uint64))
    out = torch.full((H, total, 128), float("nan"), device="cuda")
    cache.read(out)
    torch.cuda.synchronize()
    assert hq.read_stats(cache.stats)["status"] == 0
    n = sum(len(o) for o in offs) - 1
    assert_same_words(cache.words[:base].cpu().numpy().view(np.uint32),
                      cache.offsets[:n + 1].cpu().numpy().view(np.uint64), np.concatenate(words), np.concatenate(offs))
    assert_recon_equal(out.cpu().numpy(), ref)


@pytest.mark.parametrize("lat", ["E8", "D4", "A2", "Z"])
@pytest.mark.parametrize("dither", [0, 1])
def test_rotated_one_token_appends(lat, dither):
    K, V = synth.kv(8, 24, seed=41)
    _rot_case(8, [1] * 10 + [7] + [1] * 7, lat, ALPHA[lat] * 2.0, 1, seed=13, dither=dither,
              source=K if dither else V, rot_seed=5)


@pytest.mark.parametrize("H,k", [(1, 0), (17, 2), (32, 6)])
def test_rotated_head_counts(H, k):
    """Up to 32 one-tile chunks (the multi-token single-CTA form with the rotation stops at 16)."""
    K, _ = synth.kv(H, 5, seed=H + 50)
    _rot_case(H, [1] * 5, "E8", 0.35 * 2.0 ** k, k, seed=2, dither=1, source=K, rot_seed=H)


def test_rotated_forms_agree_on_one_token():
    """Grouped form (forced) and the one-token form give one stream with the rotation."""
    from oracle import rotation as R
    hq = _hq()
    K, _ = synth.kv(8, 6, seed=22)
    Q = torch.from_numpy(R.haar_rotation(9)).cuda()
    outs = []
    for path in (2, 4):
        hq.hq_debug_set_encode_path(path)
        try:
            cache = hq.KVCache(8, 6, hq.make_params("E8", 1.0, 1, 4, 1), bits_per_scalar=16.0, max_appends=7,
                               max_append_tokens=1, rotation=Q)
            for t in range(6):
                cache.append(K[:, t:t + 1].contiguous().cuda(), 0.7)
            torch.cuda.synchronize()
            end = int(cache.offsets[48].item())
            outs.append((cache.words[:end].cpu().numpy().copy(), cache.offsets[:49].cpu().numpy().copy()))
        finally:
            hq.hq_debug_set_encode_path(0)
    assert np.array_equal(outs[0][1], outs[1][1]) and np.array_equal(outs[0][0], outs[1][0])
