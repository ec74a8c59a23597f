"""Seeded random combinations of every option against the oracle.

Each case draws a lattice, a Rice parameter, a second parameter for the halved symbol,
dither, the encoder form, and a shape (weights) or a sequence of appends (KV, with or
without a dense rotation), and checks streams, offsets, stats and reconstructions.
The draws are fixed by the case number, so a failure names a reproducible case."""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import rotation as R
import synth
from hqtest import assert_recon_equal, assert_same_words, gpu_dequantize, gpu_quantize, oracle_dequantize, oracle_quantize

pytestmark = pytest.mark.gpu

LATS = ["E8", "D4", "A2", "Z"]
# alpha near 3 bps at k = 2 for the weights recipe (std 0.02), scaled by 2^(k - 2)
W_ALPHA = {"E8": 160.0, "D4": 92.0, "A2": 70.0, "Z": 78.0}
# alpha near 2 bps at k = 0 for the KV recipe (std 1), scaled by 2^k
KV_ALPHA = {"E8": 0.35, "D4": 0.3, "A2": 0.25, "Z": 0.3}


def _hq():
    import lattice_entropy_coded_b200 as hq
    return hq


@pytest.mark.parametrize("case", range(64))
def test_weights_random_options(case):
    hq = _hq()
    rng = np.random.default_rng(1000 + case)
    lat = LATS[rng.integers(4)]
    k = int(rng.integers(0, 7))
    dk = int(rng.integers(0, 4))
    dither = int(rng.integers(0, 2))
    path = int(rng.integers(0, 5))
    rows, cols = int(rng.integers(1, 90)), 128 * int(rng.integers(1, 20))
    alpha = W_ALPHA[lat] * 2.0 ** (k - 2) * float(rng.uniform(0.7, 1.4))
    seed = int(rng.integers(0, 2**63))
    x = synth.weight(rows, cols, seed=case)
    L = O.LATTICES[lat]
    p = hq.make_params(lat, alpha, k, seed, dither, dk_last=dk)
    hq.hq_debug_set_encode_path(path)
    try:
        g = gpu_quantize(x.cuda(), p, max_abs_symbol=4095)
    finally:
        hq.hq_debug_set_encode_path(0)
    ref_w, ref_off, ref_pay = oracle_quantize(x, L, alpha, k, seed, dither, dk_last=dk)
    assert g["stats"]["status"] == 0, (case, g["stats"])
    assert_same_words(g["words"], g["offsets"], ref_w, ref_off)
    assert g["stats"]["payload_bits"] == ref_pay
    y, st, _ = gpu_dequantize(g["words_t"], g["cap"], g["offsets_t"], rows, cols, p, fp32=True)
    assert st["status"] == 0
    assert_recon_equal(y, oracle_dequantize(ref_w, ref_off, rows, cols, L, alpha, k, seed, dither, fp32=True,
                                            dk_last=dk))


@pytest.mark.parametrize("case", range(48))
def test_kv_random_options(case):
    hq = _hq()
    rng = np.random.default_rng(2000 + case)
    lat = LATS[rng.integers(4)]
    k = int(rng.integers(0, 5))
    dk = int(rng.integers(0, 3))
    dither = int(rng.integers(0, 2))
    path = int(rng.integers(0, 5))
    H = int(rng.integers(1, 13))
    Ts = [int(t) for t in rng.integers(1, 120, size=int(rng.integers(1, 5)))]
    rot = bool(rng.integers(0, 2))
    alpha = KV_ALPHA[lat] * 2.0 ** k
    seed = int(rng.integers(0, 2**63))
    total = sum(Ts)
    K, V = synth.kv(H, total, seed=case)
    src = K if case % 2 else V
    Q = R.haar_rotation(case) if rot else None
    L = O.LATTICES[lat]
    cache = hq.KVCache(H, total, hq.make_params(lat, 1.0, k, seed, dither, dk_last=dk), bits_per_scalar=24.0,
                       max_appends=len(Ts) + 1, max_append_tokens=max(Ts),
                       rotation=torch.from_numpy(Q).cuda() if rot else None)
    hq.hq_debug_set_encode_path(path)
    words, offs, base, t0 = [], [], 0, 0
    ref = np.zeros((H, total, 128), np.float32)
    try:
        for T in Ts:
            a = src[:, t0:t0 + T].contiguous()
            cache.append(a.cuda(), alpha)
            s, off, _ = O.kv_append(a, t0, L, alpha, k, seed, dither, base_word=base, rot=Q, dk_last=dk)
            O.kv_read_append(s, off - np.uint64(base), H, T, t0, L, alpha, k, seed, dither, ref, total, rot=Q,
                             dk_last=dk)
            words.append(s)
            offs.append(off[:-1])
            base = int(off[-1])
            t0 += T
    finally:
        hq.hq_debug_set_encode_path(0)
    offs.append(np.array([base], np.uint64))
    out = torch.full((H, total, 128), float("nan"), device="cuda")
    cache.read(out)
    torch.cuda.synchronize()
    assert hq.read_stats(cache.stats)["status"] == 0, case
    n = sum(len(o) for o in offs) - 1
    assert_same_words(cache.words[:base].cpu().numpy().view(np.uint32),
                      cache.offsets[:n + 1].cpu().numpy().view(np.uint64), np.concatenate(words), np.concatenate(offs))
    assert_recon_equal(out.cpu().numpy(), ref)
