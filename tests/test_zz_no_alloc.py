"""hq_quantize_static: the quantize entry point for callers that cannot allocate
device memory (a plug-in inside a host that owns every allocation, or a path
where cudaMalloc is not allowed).  Its scratch is a fixed array inside
libhq.so, so it must give exactly what hq_quantize gives with a caller
workspace -- on two calls in a row, since the second call finds the first
call's look-back state in that array and must clear it.

This file is collected last on purpose; it passes alone in a fresh process and
after the rest of the suite."""
import ctypes as C

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


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


@pytest.mark.parametrize("lattice,alpha,k,dither,shape", [
    ("E8", 314.15, 2, 0, (37, 384)),       # ragged last chunk
    ("D4", 183.8, 2, 1, (256, 4096)),      # dither
    ("Z", 160.7, 2, 0, (1024, 1024)),
])
def test_static_scratch_matches_workspace_entry_point(lattice, alpha, k, dither, shape):
    import lattice_entropy_coded_b200 as hq
    params = hq.make_params(lattice, alpha, k, 5, dither)
    x = synth.weight(*shape, seed=21).cuda()
    cap, nch = hq.hq_stream_bound(shape[0], shape[1], params)
    ref_words = torch.full((cap,), 7, dtype=torch.int32, device="cuda")
    ref_off = torch.full((nch + 1,), -1, dtype=torch.int64, device="cuda")
    ref_stats = hq.stats_tensor("cuda")
    ws = torch.empty(hq.hq_workspace_bytes(nch), dtype=torch.uint8, device="cuda")
    hq.hq_quantize(x, params, ref_words, ref_off, ref_stats, ws)
    torch.cuda.synchronize()
    ref = hq.read_stats(ref_stats)
    assert ref["status"] == 0
    total = int(ref_off[-1].item())
    for call in range(2):
        words, offsets, st = _run_static(hq, x, params, cap, nch)
        assert st == ref, f"call {call}"
        assert torch.equal(offsets, ref_off), f"call {call}"
        assert torch.equal(words[:total], ref_words[:total]), f"call {call}"
        # stream words decode to the same reconstruction as well
        out = torch.empty(shape, dtype=torch.float32, device="cuda")
        hq.hq_dequantize(words, cap, offsets, shape[0], shape[1], params, out)
        ref_out = torch.empty(shape, dtype=torch.float32, device="cuda")
        hq.hq_dequantize(ref_words, cap, ref_off, shape[0], shape[1], params, ref_out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out)


def test_static_scratch_rejects_sizes_beyond_its_limit():
    import lattice_entropy_coded_b200 as hq
    params = hq.make_params("E8", 300.0, 2, 0, 0)
    too_many_rows = (131067 * 32 + 32) // 32 + 1          # cols = 4096: one chunk per row
    x = torch.empty(1, 4096, dtype=torch.bfloat16, device="cuda")
    rc = hq._lib.hq_quantize_static(x.data_ptr(), too_many_rows, 4096, 4096, C.byref(params), x.data_ptr(), 0,
                                    x.data_ptr(), None, None)
    assert rc == hq.HQ_EUNSUPPORTED
