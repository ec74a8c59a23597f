"""Rate targeting on the device against the quantize path and the oracle.

hq_rate must report exactly the stats hq_quantize reports for the same call (payload
bits, stream words, largest symbol); hq_rate_kv exactly the payload of the same
tokens appended to a KV cache in any split.  hq_calibrate runs the bisection of
tests/golden/calibrate_points.py on the device; fed the same (bit-exact) rates it
must land on the same alpha and k as that script does with the oracle.
"""
import importlib.util
import os

import numpy as np
import pytest
import torch

import oracle as O
import synth
from hqtest import GOLD, gpu_quantize, oracle_quantize, u16

pytestmark = pytest.mark.gpu


def _hq():
    import lattice_entropy_coded_b200 as hq
    return hq


def _calibration_script():
    spec = importlib.util.spec_from_file_location("calibrate_points", os.path.join(GOLD, "calibrate_points.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("lat", ["E8", "D4", "A2", "Z"])
@pytest.mark.parametrize("dither", [0, 1])
@pytest.mark.parametrize("shape,k,alpha", [((37, 384), 2, 300.0), ((64, 4096), 1, 150.0), ((5, 1152), 5, 4000.0)])
def test_rate_equals_quantize_stats(lat, dither, shape, k, alpha):
    hq = _hq()
    x = synth.weight(*shape, seed=21 + shape[0]).cuda()
    p = hq.make_params(lat, alpha, k, 99, dither)
    g = gpu_quantize(x, p, max_abs_symbol=1 << 14)
    st = hq.stats_tensor()
    hq.hq_rate(x, p, st)
    r = hq.read_stats(st)
    assert r["status"] == g["stats"]["status"] == 0
    assert r["payload_bits"] == g["stats"]["payload_bits"]
    assert r["stream_words"] == g["stats"]["stream_words"] == g["total"]
    assert r["max_symbol"] == g["stats"]["max_symbol"]


def test_rate_equals_oracle_payload_full_matrix():
    hq = _hq()
    x = synth.weight(1024, 1024, seed=0)
    p = hq.make_params("E8", 313.2163391113281, 2, 0, 0)
    st = hq.stats_tensor()
    hq.hq_rate(x.cuda(), p, st)
    ref_w, ref_off, ref_pay = oracle_quantize(x, O.E8, 313.2163391113281, 2, 0)
    r = hq.read_stats(st)
    assert r["payload_bits"] == ref_pay and r["stream_words"] == len(ref_w)


@pytest.mark.parametrize("lat", ["E8", "Z"])
def test_rate_kv_equals_appends(lat):
    hq = _hq()
    H = 4
    K, _ = synth.kv(H, 300, seed=3)
    params = hq.make_params(lat, 1.0, 1, 5, 1)
    cache = hq.KVCache(H, 300, params, bits_per_scalar=16.0, max_appends=8, max_append_tokens=256)
    t0 = 0
    for T in (100, 1, 199):
        cache.append(K[:, t0:t0 + T].contiguous().cuda(), 0.4)
        t0 += T
    appended = hq.read_stats(cache.stats)["payload_bits"]
    st = hq.stats_tensor()
    hq.hq_rate_kv(K.cuda(), hq.make_params(lat, 0.4, 1, 5, 1), st, tok0=0)
    assert hq.read_stats(st)["payload_bits"] == appended
    # a block at a later position uses that position's dither
    hq.hq_rate_kv(K[:, 100:].contiguous().cuda(), hq.make_params(lat, 0.4, 1, 5, 1), st, tok0=100)
    _, _, pay = O.kv_append(u16(K[:, 100:].contiguous()), 100, O.LATTICES[lat], 0.4, 1, 5, 1)
    assert hq.read_stats(st)["payload_bits"] == pay


def test_calibrate_matches_the_oracle_bisection():
    hq = _hq()
    cp = _calibration_script()
    x = synth.weight(64, 1024, seed=1)
    xu = u16(x)
    for lat, target, ks in (("E8", 4.0, (1, 3)), ("D4", 3.0, (0, 2)), ("Z", 5.0, (2, 4))):
        L = O.LATTICES[lat]
        want = cp.calibrate(lambda a, k: cp.weight_bits(xu, L, a, k, 7) / xu.size, target, range(ks[0], ks[1] + 1))
        got = hq.hq_calibrate(x.cuda(), hq.make_params(lat, 1.0, 0, 7, 0), hq.calib_spec(target, k_lo=ks[0], k_hi=ks[1]),
                              hq.stats_tensor())
        assert got["k"] == want["k"], (lat, got, want)
        assert np.float32(got["alpha"]) == np.float32(want["alpha"]), (lat, got, want)
        assert got["bps"] == want["bps_payload_sample"], (lat, got, want)
        assert abs(got["bps"] - target) <= 0.002 and got["status"] == 0


def test_calibrate_kv_matches_the_oracle_bisection():
    hq = _hq()
    cp = _calibration_script()
    K, _ = synth.kv(2, 96, seed=4)
    ku = u16(K)
    want = cp.calibrate(lambda a, k: O.kv_append(ku, 0, O.E8, a, k, 9, 1)[2] / ku.size, 2.0, range(0, 2))
    got = hq.hq_calibrate_kv(K.cuda(), hq.make_params("E8", 1.0, 0, 9, 1), hq.calib_spec(2.0, k_lo=0, k_hi=1),
                             hq.stats_tensor())
    assert got["k"] == want["k"] and np.float32(got["alpha"]) == np.float32(want["alpha"])
    assert got["bps"] == want["bps_payload_sample"]


def test_calibrate_reports_an_unreachable_target():
    hq = _hq()
    x = synth.weight(8, 256, seed=2).cuda()
    with pytest.raises(hq.HQError):
        hq.hq_calibrate(x, hq.make_params("E8", 1.0, 0, 1, 0), hq.calib_spec(4.0, alpha_lo=1e-3, alpha_hi=1e-2),
                        hq.stats_tensor())
