"""hq_quantize_static: the quantize entry point for callers that cannot allocate
device memory (a plug-in inside a host that owns every allocation, or a path
where cudaMalloc is not allowed).  Its scratch is a fixed array inside
libhq.so, so it must give exactly what hq_quantize gives with a caller
workspace -- on two calls in a row, since the second call finds the first
call's look-back state in that array and must clear it.  Every encoder form
runs with the array (forced in turn), a large call is followed by a smaller
one (stale look-back words beyond the second call's chunks), and one call sits
at the array's chunk limit.

This file is collected last on purpose; it passes alone in a fresh process and
after the rest of the suite."""
import ctypes as C

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _hq():
    import lattice_entropy_coded_b200 as hq
    return hq


def _run_static(hq, x, params, cap, nch):
    words = torch.full((cap,), 7, dtype=torch.int32, device="cuda")
    offsets = torch.full((nch + 1,), -1, dtype=torch.int64, device="cuda")
    stats = hq.stats_tensor("cuda")
    rc = hq._lib.hq_quantize_static(x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), C.byref(params),
                                    words.data_ptr(), cap, offsets.data_ptr(), stats.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    assert rc == hq.HQ_OK
    torch.cuda.synchronize()
    return words, offsets, hq.read_stats(stats)


def _run_workspace(hq, x, params, cap, nch):
    words = torch.full((cap,), 7, dtype=torch.int32, device="cuda")
    offsets = torch.full((nch + 1,), -1, dtype=torch.int64, device="cuda")
    stats = hq.stats_tensor("cuda")
    ws = torch.empty(hq.hq_workspace_bytes(nch), dtype=torch.uint8, device="cuda")
    hq.hq_quantize(x, params, words, offsets, stats, ws)
    torch.cuda.synchronize()
    return words, offsets, hq.read_stats(stats)


def _check_against_workspace(hq, x, params, calls=2, decode=True, max_abs_symbol=0):
    rows, cols = x.shape
    cap, nch = hq.hq_stream_bound(rows, cols, params, max_abs_symbol)
    ref_words, ref_off, ref = _run_workspace(hq, x, params, cap, nch)
    assert ref["status"] == 0
    total = int(ref_off[-1].item())
    for call in range(calls):
        words, offsets, st = _run_static(hq, x, params, cap, nch)
        assert st == ref, f"call {call}"
        assert torch.equal(offsets, ref_off), f"call {call}"
        assert torch.equal(words[:total], ref_words[:total]), f"call {call}"
        if decode:
            # the stream decodes to the same reconstruction as well
            out = torch.empty(rows, cols, dtype=torch.float32, device="cuda")
            hq.hq_dequantize(words, cap, offsets, rows, cols, params, out)
            ref_out = torch.empty(rows, cols, dtype=torch.float32, device="cuda")
            hq.hq_dequantize(ref_words, cap, ref_off, rows, cols, params, ref_out)
            torch.cuda.synchronize()
            assert torch.equal(out, ref_out)


@pytest.fixture(params=[0, 1, 2, 3, 4], ids=["by_size", "per_warp", "grouped", "wide", "single_cta"])
def path(request):
    hq = _hq()
    hq.hq_debug_set_encode_path(request.param)
    yield request.param
    hq.hq_debug_set_encode_path(0)


@pytest.mark.parametrize("lattice,alpha,k,dither,shape", [
    ("E8", 314.15, 2, 0, (37, 384)),       # ragged last chunk
    ("D4", 183.8, 2, 1, (256, 4096)),      # dither
    ("Z", 160.7, 2, 0, (1024, 1024)),
])
def test_static_scratch_matches_workspace_entry_point(path, lattice, alpha, k, dither, shape):
    hq = _hq()
    params = hq.make_params(lattice, alpha, k, 5, dither)
    x = synth.weight(*shape, seed=21).cuda()
    _check_against_workspace(hq, x, params)


def test_large_call_then_small_call():
    """A 4096 x 4096 call (4096 chunks, the per-warp form) leaves look-back words for
    chunks the following 1024 x 1024 call (256 chunks) does not use; both match."""
    hq = _hq()
    params = hq.make_params("E8", 314.15, 2, 1, 0)
    big = synth.weight(4096, 4096, seed=1).cuda()
    small = synth.weight(1024, 1024, seed=0).cuda()
    _check_against_workspace(hq, big, params, calls=1)
    _check_against_workspace(hq, small, params, calls=2)
    _check_against_workspace(hq, big, params, calls=1)


def test_call_at_the_chunk_limit():
    """HQ_STATIC_MAX_CHUNKS chunks (rows of 4096 elements: one chunk per row), the
    largest call the fixed scratch holds (one more row is refused, below).  The stream
    bound assumes symbols up to 64 (the Gaussian codes here stay far below it)."""
    hq = _hq()
    rows = hq.HQ_STATIC_MAX_CHUNKS
    params = hq.make_params("E8", 314.15, 2, 2, 0)
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    x = (torch.randn(rows, 4096, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    _check_against_workspace(hq, x, params, calls=2, decode=False, max_abs_symbol=64)
    del x
    torch.cuda.empty_cache()


def test_static_scratch_rejects_sizes_beyond_its_limit():
    """Beyond the limit the call returns HQ_EUNSUPPORTED before looking at any pointer
    (all null here, so nothing could reach the device)."""
    hq = _hq()
    params = hq.make_params("E8", 300.0, 2, 0, 0)
    rc = hq._lib.hq_quantize_static(None, hq.HQ_STATIC_MAX_CHUNKS + 1, 4096, 4096, C.byref(params), None, 0, None,
                                    None, None)
    assert rc == hq.HQ_EUNSUPPORTED
