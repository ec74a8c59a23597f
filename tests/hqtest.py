"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
(via the binding) and the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import json
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle as O

POISON = 0xDEADBEEF          # fill of stream buffers: words nobody wrote keep it
GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
THREADS = max(1, min(32, os.cpu_count() or 1))
_POOL = ThreadPoolExecutor(THREADS)


def rate_points():
    with open(os.path.join(GOLD, "rate_points.json")) as f:
        return json.load(f)["workloads"]


def u16(t: torch.Tensor) -> np.ndarray:
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


# ---------------------------------------------------------------- oracle (threaded over chunk ranges)
def oracle_quantize(x: torch.Tensor, lat: int, alpha: float, k: int, seed: int, dither: int = 0, dk_last: int = 0):
    """-> (words uint32 [total], offsets uint64 [n+1] absolute, payload bits)."""
    xu = u16(x)
    R, Cc = xu.shape
    nch = O.n_chunks(R, Cc)
    if nch == 0:
        return np.zeros(0, np.uint32), np.zeros(1, np.uint64), 0
    step = max(1, -(-nch // THREADS))
    ranges = [(a, min(nch, a + step)) for a in range(0, nch, step)]
    parts = list(_POOL.map(lambda r: O.quantize(xu, lat, alpha, k, seed, dither, r[0], r[1], dk_last=dk_last), ranges))
    words, offs, pay, base = [], [], 0, 0
    for (s, off, pb) in parts:
        words.append(s[:int(off[-1])])
        offs.append(off[:-1].astype(np.uint64) + np.uint64(base))
        base += int(off[-1])
        pay += pb
    offs.append(np.array([base], np.uint64))
    return np.concatenate(words), np.concatenate(offs), pay


def oracle_dequantize(words, offsets, rows, cols, lat, alpha, k, seed, dither=0, fp32=True, dk_last=0):
    out = np.zeros((rows, cols), np.float32 if fp32 else np.uint16)
    nch = len(offsets) - 1
    if nch == 0:
        return out
    step = max(1, -(-nch // THREADS))
    ranges = [(a, min(nch, a + step)) for a in range(0, nch, step)]
    list(_POOL.map(lambda r: O.dequantize(words, offsets[r[0]:r[1] + 1], rows, cols, lat, alpha, k, seed, dither,
                                          fp32, r[0], r[1], out=out, dk_last=dk_last), ranges))
    return out


def oracle_chunk(x: torch.Tensor, c: int, lat, alpha, k, seed, dither=0):
    """Words of chunk c alone (the oracle computes any chunk on its own)."""
    s, off, pb = O.quantize(u16(x), lat, alpha, k, seed, dither, c, c + 1)
    return s[:int(off[1])], pb


# ---------------------------------------------------------------- CUDA path
def gpu_quantize(x: torch.Tensor, params, cap_words: int | None = None, guard: int = 0, ld: int | None = None,
                 max_abs_symbol: int = 0):
    """x on the GPU (bf16).  -> dict(words np [total], offsets np, stats, words_t, offsets_t, cap)."""
    import lattice_entropy_coded_b200 as hq
    rows, cols = x.shape
    bound, nch = hq.hq_stream_bound(rows, cols, params, max_abs_symbol)
    cap = bound if cap_words is None else cap_words
    words = torch.full((cap + guard + 1,), POISON - (1 << 32), dtype=torch.int32, device=x.device)
    offsets = torch.full((nch + 1,), -1, dtype=torch.int64, device=x.device)
    stats = hq.stats_tensor(x.device)
    ws = torch.empty(hq.hq_workspace_bytes(nch), dtype=torch.uint8, device=x.device)
    hq.hq_quantize(x, params, words[:cap], offsets, stats, ws, ld=ld)
    torch.cuda.synchronize()
    st = hq.read_stats(stats)
    off = offsets.cpu().numpy().view(np.uint64)
    total = int(off[-1]) if nch else 0
    w = words.cpu().numpy().view(np.uint32)
    return dict(words=w[:min(total, cap)], all_words=w, offsets=off, stats=st, words_t=words, offsets_t=offsets,
                cap=cap, total=total)


def gpu_dequantize(words_t: torch.Tensor, stream_words: int, offsets_t: torch.Tensor, rows: int, cols: int, params,
                   fp32: bool = True, ld: int | None = None):
    import lattice_entropy_coded_b200 as hq
    ld = cols if ld is None else ld
    buf = torch.full((rows, ld), float("nan"), dtype=torch.float32 if fp32 else torch.bfloat16,
                     device=words_t.device)
    out = buf[:, :cols]
    stats = hq.stats_tensor(words_t.device)
    hq.hq_dequantize(words_t, stream_words, offsets_t, rows, cols, params, out, stats)
    torch.cuda.synchronize()
    res = out.cpu()
    if fp32:
        res = res.numpy()
    else:
        res = res.contiguous().view(torch.int16).numpy().view(np.uint16)
    return res, hq.read_stats(stats), buf


def assert_same_words(gpu_words: np.ndarray, gpu_offsets: np.ndarray, ref_words: np.ndarray, ref_offsets: np.ndarray):
    assert np.array_equal(gpu_offsets.astype(np.uint64), ref_offsets.astype(np.uint64)), "chunk offsets differ"
    if not np.array_equal(gpu_words, ref_words):
        bad = np.nonzero(gpu_words != ref_words)[0]
        i = int(bad[0])
        c = int(np.searchsorted(ref_offsets, i, side="right") - 1)
        raise AssertionError(f"{len(bad)} stream words differ; first at word {i} (chunk {c}): "
                             f"gpu {gpu_words[i]:#010x} oracle {ref_words[i]:#010x}")


def assert_recon_equal(gpu: np.ndarray, ref: np.ndarray, rel: float = 1e-6):
    """fp32 reconstructions: within rel * max(1, |ref|) per element (the bar); they are
    expected to be bit-identical, and bit-identity is reported when it holds."""
    g = gpu.astype(np.float64)
    r = ref.astype(np.float64)
    err = np.abs(g - r)
    lim = rel * np.maximum(np.abs(r), 1e-30)
    bad = err > lim
    assert not bad.any(), f"{int(bad.sum())} elements differ beyond {rel} relative; worst {float(err.max())}"
