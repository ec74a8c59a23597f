"""The integer range of the codes (hq_stats.max_abs_code, int8_overflow_count) on the
GPU against the oracle, through the C ABI.

The pages store the lattice points' integers in 8 bits with alpha calibrated so
that they do not overflow (explainer pages, "Methodology" 2, the integer
implementation); the encoders report the largest |code coordinate| and the count
outside [-128, 127].  Every encoder form reports them (forced in turn), as do the
rate pass and a KV cache's running stats (sign diagonal, dense rotation, and the
one-token append form).  Alphas are chosen so that some cases overflow int8 and
some do not.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from hqtest import gpu_quantize

pytestmark = pytest.mark.gpu

ALPHA_UNIT = float(np.float32(np.sqrt(128.0)))


def _hq():
    import lattice_entropy_coded_b200 as hq
    return hq


def _rng(st):
    return st["max_abs_code"], st["int8_overflow_count"]


@pytest.fixture(params=[0, 1, 2, 3, 4], ids=["by_size", "per_warp", "grouped", "wide", "single_cta"])
def path(request):
    hq = _hq()
    hq.hq_debug_set_encode_path(request.param)
    yield request.param
    hq.hq_debug_set_encode_path(0)


@pytest.mark.parametrize("lat,alpha", [("E8", 3000.0), ("E8", 314.15), ("D4", 2000.0), ("A2", 2500.0),
                                       ("Z", 2000.0)])
@pytest.mark.parametrize("dither", [0, 1])
def test_weights_range_matches_oracle(path, lat, alpha, dither):
    hq = _hq()
    for shape in ((37, 384), (64, 4096)):
        x = synth.weight(*shape, seed=31)
        p = hq.make_params(lat, alpha, 3, 7, dither)
        g = gpu_quantize(x.cuda(), p)
        want = O.quantize_range(x, O.LATTICES[lat], alpha, 7, dither)
        assert g["stats"]["status"] == 0
        assert _rng(g["stats"]) == want, (shape, g["stats"], want)
        st = hq.stats_tensor()
        hq.hq_rate(x.cuda(), p, st)
        torch.cuda.synchronize()
        assert _rng(hq.read_stats(st)) == want


def test_range_at_the_int8_edges():
    """One-hot rows with a unit forward scale: codes are exactly +-value (closed form),
    with values at and around both ends of int8."""
    hq = _hq()
    vals = [5.0, -5.0, 127.0, -127.0, 128.0, -128.0, 129.0, -129.0, 200.0, -200.0]
    x = torch.zeros(len(vals), 256)
    x[:, 0] = torch.tensor(vals)
    x = x.to(torch.bfloat16)
    for lat in ("E8", "D4", "Z"):
        p = hq.make_params(lat, ALPHA_UNIT, 3, 3, 0)
        g = gpu_quantize(x.cuda(), p)
        want = O.quantize_range(x, O.LATTICES[lat], ALPHA_UNIT, 3)
        assert want[0] == 200
        assert _rng(g["stats"]) == want


def test_large_matrix_range():
    """4096 x 4096 at E8: the per-warp form by size, with and without overflow."""
    hq = _hq()
    x = synth.weight(4096, 4096, seed=1)
    xg = x.cuda()
    for alpha in (314.15, 2500.0):
        p = hq.make_params("E8", alpha, 2, 1, 0)
        g = gpu_quantize(xg, p, cap_words=int(x.numel() * 12 // 32) + 65536)
        want = O.quantize_range(x, O.E8, alpha, 1)
        assert _rng(g["stats"]) == want


@pytest.mark.parametrize("rot", [False, True])
def test_kv_running_range(rot):
    """A KV cache's stats keep the maximum and the sum over appends: appends of 40,
    1 (the one-token form) and 300 tokens, E8 with dither, large enough alpha to
    overflow int8 in places."""
    hq = _hq()
    from oracle import rotation as ORot
    K, _ = synth.kv(3, 341, seed=4)
    seed, alpha, k = 6, 9.0, 2
    Q = ORot.haar_rotation(seed) if rot else None
    cache = hq.KVCache(3, 341, hq.make_params("E8", 1.0, k, seed, 1), bits_per_scalar=64.0, max_appends=4,
                       max_append_tokens=300, rotation=torch.from_numpy(Q).cuda() if rot else None)
    mx, ov = 0, 0
    t0 = 0
    for T in (40, 1, 300):
        blk = K[:, t0:t0 + T].contiguous()
        cache.append(blk.cuda(), alpha)
        m, o = O.kv_range(blk, t0, O.E8, alpha, seed, 1, rot=Q)
        mx, ov = max(mx, m), ov + o
        t0 += T
    torch.cuda.synchronize()
    st = hq.read_stats(cache.stats)
    assert st["status"] == 0
    assert ov > 0
    assert _rng(st) == (mx, ov)
    # the rate pass over the same tokens reports the same range
    st2 = hq.stats_tensor()
    p = hq.make_params("E8", alpha, k, seed, 1)
    if rot:
        p.rotation = cache.rotation.data_ptr()
    hq.hq_rate_kv(K.cuda(), p, st2)
    torch.cuda.synchronize()
    assert _rng(hq.read_stats(st2)) == O.kv_range(K, 0, O.E8, alpha, seed, 1, rot=Q)


def test_decode_leaves_range_zero():
    hq = _hq()
    x = synth.weight(64, 512, seed=2)
    p = hq.make_params("E8", 3000.0, 3, 1, 0)
    g = gpu_quantize(x.cuda(), p)
    assert g["stats"]["int8_overflow_count"] > 0
    st = hq.stats_tensor()
    out = torch.empty(64, 512, device="cuda")
    hq.hq_dequantize(g["words_t"], g["cap"], g["offsets_t"], 64, 512, p, out, st)
    torch.cuda.synchronize()
    assert _rng(hq.read_stats(st)) == (0, 0)


@pytest.mark.parametrize("lat,alpha,dither", [("E8", 3000.0, 0), ("E8", 314.15, 1), ("D4", 2000.0, 0),
                                              ("A2", 2500.0, 1), ("Z", 700.0, 0)])
def test_max_symbol_is_the_or_of_all_symbols(path, lat, alpha, dither):
    """hq_stats.max_symbol is the bitwise OR of every zigzag symbol of the call (its bit
    length bounds them all, the figure hq_stream_bound's max_abs_symbol takes): every chunk
    of the oracle's stream decoded back to codes, each lattice block stripped to its symbols
    by the oracle, and the OR taken."""
    hq = _hq()
    L = O.LATTICES[lat]
    n = O.DIM[L]
    for rows, cols in ((37, 384), (64, 1024)):
        x = synth.weight(rows, cols, seed=33)
        p = hq.make_params(lat, alpha, 3, 9, dither)
        g = gpu_quantize(x.cuda(), p)
        s, off, _ = O.quantize(x, L, alpha, 3, 9, dither)
        want = 0
        for c in range(O.n_chunks(rows, cols)):
            nt = min(32, rows * cols // 128 - 32 * c)
            q = O.decode_chunk(L, 3, s[int(off[c]):int(off[c + 1])], nt)
            for b in range(q.size // n):
                m, _ = O.strip(L, q[b * n:(b + 1) * n])
                for v in m:
                    want |= O.zigzag(int(v))
        assert g["stats"]["status"] == 0
        assert g["stats"]["max_symbol"] == want, (rows, cols, g["stats"]["max_symbol"], want)
