"""Every form of the quantize kernel against the oracle.

The encoder has a per-warp form (a warp encodes whole chunks; used for large
launches), a grouped form (four warps share a chunk), a wide form (sixteen warps
share a chunk) and a single-CTA form (one CTA for a launch of at most 32 chunks,
such as a KV append of a few tokens; forced on a larger launch, the per-warp form
runs).  The per-warp form takes its input by one bulk copy per round where the
rows hold whole rounds (cols a multiple of 1024: the 4096 and 65536 column cases)
and by per-lane copies otherwise (384 columns, strided rows).  By default the size decides;
here each form is forced in turn on the cases that exercise its control flow:
ragged last chunks, every Rice parameter, strided rows, exact ties, chunks too
large for the shared stage, capacity overflow, bounded look-back waits, KV
appends, and a 4096 x 4096 matrix (many chunks per group or warp).
"""
import numpy as np
import pytest

import oracle as O
import synth
import test_gpu_parity as P
from hqtest import assert_same_words, gpu_quantize, oracle_quantize, rate_points

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[1, 2, 3, 4], ids=["per_warp", "grouped", "wide", "single_cta"])
def path(request):
    import lattice_entropy_coded_b200 as hq
    hq.hq_debug_set_encode_path(request.param)
    yield request.param
    hq.hq_debug_set_encode_path(0)


@pytest.mark.parametrize("lat", ["E8", "D4", "A2", "Z"])
@pytest.mark.parametrize("dither", [0, 1])
def test_small_matrices(path, lat, dither):
    P.test_weights_bit_exact_small(lat, dither, (37, 384))
    P.test_weights_bit_exact_small(lat, dither, (64, 4096))
    P.test_weights_bit_exact_small(lat, dither, (3, 65536))    # the widest rows (512 tile columns)


@pytest.mark.parametrize("k", [0, 3, 8, 15])
def test_rice_parameters(path, k):
    P.test_every_rice_parameter(k)


def test_strided_ties_zero(path):
    P.test_strided_rows()
    P.test_all_zero_and_tiny_alpha()
    P.test_ties_and_structured_inputs()


def test_stage_overflow_slow_path(path):
    P.test_large_symbols_take_the_slow_path_with_the_same_bits()


def test_capacity_and_timeouts(path):
    P.test_capacity_overflow_is_flagged_and_bounded()
    P.test_lookback_spin_limit_never_hangs()
    P.test_empty_matrix()


@pytest.mark.parametrize("lat", ["E8", "Z"])
def test_kv_appends(path, lat):
    P.test_kv_appends_bit_exact(lat)


def test_kv_appends_k0(path):
    P.test_kv_appends_k0_bit_exact()


def test_many_chunks_per_worker(path):
    """4096 x 4096 (4096 chunks): every group or warp encodes several chunks in turn."""
    import lattice_entropy_coded_b200 as hq
    x = synth.weight(4096, 4096, seed=1)
    p = [q for q in rate_points()["weight_4096x4096_rate_sweep"]["points"]
         if q["lattice"] == "E8" and q["bps"] == 4.0][0]
    params = hq.make_params(O.E8, p["alpha"], p["k"], 1, 0)
    g = gpu_quantize(x.cuda(), params)
    ref_w, ref_off, ref_pay = oracle_quantize(x, O.E8, p["alpha"], p["k"], 1)
    assert g["stats"]["status"] == 0
    assert_same_words(g["words"], g["offsets"], ref_w, ref_off)
    assert g["stats"]["payload_bits"] == ref_pay
    assert np.uint64(g["stats"]["stream_words"]) == ref_off[-1]


def test_stats_are_replaced_not_accumulated(path):
    """hq_quantize's stats block is written by the kernel's last CTA: whatever it held
    before (here all bytes 0xFF) is replaced by exactly this call's stats."""
    import torch
    import lattice_entropy_coded_b200 as hq
    x = synth.weight(64, 4096, seed=13).cuda()
    params = hq.make_params("E8", 300.0, 2, 1, 0)
    ref = gpu_quantize(x, params)
    bound, nch = hq.hq_stream_bound(64, 4096, params)
    words = torch.empty(bound, dtype=torch.int32, device="cuda")
    offs = torch.empty(nch + 1, dtype=torch.int64, device="cuda")
    ws = torch.empty(hq.hq_workspace_bytes(nch), dtype=torch.uint8, device="cuda")
    st = torch.full((hq.STATS_BYTES,), 0xFF, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        hq.hq_quantize(x, params, words, offs, st, ws)
        got = hq.read_stats(st)
        assert got == ref["stats"], (got, ref["stats"])


@pytest.mark.parametrize("chunks,lat,dither,dk", [(296, "E8", 0, 0), (297, "E8", 0, 0), (1776, "E8", 0, 0),
                                                  (1777, "E8", 0, 0), (2368, "D4", 1, 0), (2369, "D4", 1, 0),
                                                  (1500, "A2", 0, 1)])
def test_default_form_boundaries(chunks, lat, dither, dk):
    """The size rule's boundaries on a B200 (wide up to 296 chunks; grouped up to 1776, or 2368
    with dither; per-warp above), on R x 4096 matrices (one chunk per row), default form."""
    import lattice_entropy_coded_b200 as hq
    alpha = {q["lattice"]: q["alpha"] for q in rate_points()["weight_4096x4096_rate_sweep"]["points"]
             if q["bps"] == 4.0}[lat]
    x = synth.weight(chunks, 4096, seed=chunks)
    params = hq.make_params(lat, alpha, 2, 3, dither, dk_last=dk)
    g = gpu_quantize(x.cuda(), params)
    ref_w, ref_off, ref_pay = oracle_quantize(x, O.LATTICES[lat], alpha, 2, 3, dither, dk_last=dk)
    assert g["stats"]["status"] == 0
    assert_same_words(g["words"], g["offsets"], ref_w, ref_off)
    assert g["stats"]["payload_bits"] == ref_pay
