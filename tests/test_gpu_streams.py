"""The library under the ways callers run it: captured in a CUDA graph and replayed,
on two streams at once, on a non-default stream.  Streams must stay bit-identical
to the plain call (and so to the oracle, which the parity tests compare)."""
import numpy as np
import pytest
import torch

import synth
from hqtest import gpu_quantize

pytestmark = pytest.mark.gpu


def _hq():
    import lattice_entropy_coded_b200 as hq
    return hq


def test_graph_capture_replays_bit_exactly():
    hq = _hq()
    x = synth.weight(512, 4096, seed=51).cuda()
    p = hq.make_params("E8", 314.0, 2, 3, 0)
    ref = gpu_quantize(x, p)
    codec = hq.Codec(512, 4096, p)
    out = torch.empty(512, 4096, dtype=torch.bfloat16, device="cuda")
    ref_out = torch.empty_like(out)
    codec.dequantize(codec.quantize(x), ref_out)         # warm-up: launch plans cached before capture
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            comp = codec.quantize(x)
            codec.dequantize(comp, out)
    for _ in range(3):
        codec.words.fill_(-1)
        out.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(codec.words[:ref["total"]].cpu().numpy().view(np.uint32), ref["words"])
        assert hq.read_stats(codec.stats) == ref["stats"]
        assert torch.equal(out, ref_out)


def test_two_streams_at_once():
    hq = _hq()
    xs = [synth.weight(2048, 4096, seed=60 + i).cuda() for i in range(2)]
    ps = [hq.make_params("E8", 314.0, 2, 3, 0), hq.make_params("D4", 183.8, 2, 4, 0)]
    refs = [gpu_quantize(x, p) for x, p in zip(xs, ps)]
    codecs = [hq.Codec(2048, 4096, p) for p in ps]
    streams = [torch.cuda.Stream() for _ in range(2)]
    torch.cuda.synchronize()
    for _ in range(3):
        for c, x, s in zip(codecs, xs, streams):
            with torch.cuda.stream(s):
                c.quantize(x, cuda_stream=s)
        torch.cuda.synchronize()
        for c, r in zip(codecs, refs):
            assert np.array_equal(c.words[:r["total"]].cpu().numpy().view(np.uint32), r["words"])
            assert np.array_equal(c.offsets.cpu().numpy().view(np.uint64), r["offsets"])


def test_kv_cache_on_a_side_stream():
    hq = _hq()
    K, _ = synth.kv(4, 200, seed=70)
    params = hq.make_params("E8", 1.0, 1, 5, 1)
    caches = [hq.KVCache(4, 200, params, bits_per_scalar=16.0, max_appends=4, max_append_tokens=128)
              for _ in range(2)]
    s = torch.cuda.Stream()
    for i, cache in enumerate(caches):
        ctx = torch.cuda.stream(s) if i else torch.cuda.stream(torch.cuda.current_stream())
        with ctx:
            for t0 in (0, 128):
                cache.append(K[:, t0:t0 + 128 if t0 == 0 else 200].contiguous().cuda(), 0.4,
                             cuda_stream=s if i else None)
    torch.cuda.synchronize()
    a, b = (hq.read_stats(c.stats) for c in caches)
    assert a == b and a["status"] == 0
    n = int(caches[0].tail[0].item())   # two appends: the tail is back in word 0
    assert np.array_equal(caches[0].words[:n].cpu().numpy(), caches[1].words[:n].cpu().numpy())
