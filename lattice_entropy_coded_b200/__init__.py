"""Python binding of libhq.so, the B200 (sm_100a) HyperQuant codec library.

Argument marshalling only: every step of the quantize / encode / decode path
runs in the library's CUDA kernels.  PyTorch supplies device memory and the
current CUDA stream.  The functions carry the C entry points' names (see
include/hq.h for the contract of each); the small classes at the end allocate
buffers with torch and call them.

There is no fallback: if libhq.so is missing or cannot be loaded, importing
the binding raises.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhq.so")

HQ_Z, HQ_A2, HQ_D4, HQ_E8 = 0, 1, 2, 3
LATTICES = {"Z": HQ_Z, "A2": HQ_A2, "D4": HQ_D4, "E8": HQ_E8}
HQ_OK, HQ_EINVAL, HQ_EUNSUPPORTED, HQ_ECUDA = 0, -1, -2, -3
HQ_ST_CAPACITY, HQ_ST_CORRUPT, HQ_ST_TIMEOUT, HQ_ST_RANGE = 1, 2, 4, 8
HQ_STATIC_MAX_CHUNKS = 131066     # include/hq.h: chunks hq_quantize_static's fixed scratch holds


class hq_params(C.Structure):
    _fields_ = [("tile", C.c_int32), ("lattice", C.c_int32), ("alpha", C.c_float), ("rice_k", C.c_int32),
                ("seed", C.c_uint64), ("dither", C.c_int32), ("chunk_tiles", C.c_int32), ("rotation", C.c_void_p),
                ("rice_dk_last", C.c_int32), ("reserved", C.c_int32)]


class hq_stats(C.Structure):
    _fields_ = [("status", C.c_uint32), ("max_symbol", C.c_uint32), ("payload_bits", C.c_uint64),
                ("stream_words", C.c_uint64), ("max_abs_code", C.c_uint32), ("reserved", C.c_uint32),
                ("int8_overflow_count", C.c_uint64)]


class hq_kv_append_row(C.Structure):
    _fields_ = [("first_chunk", C.c_uint64), ("token0", C.c_int64), ("tokens", C.c_int32), ("alpha", C.c_float),
                ("scale_fwd", C.c_float), ("scale_inv", C.c_float)]


class hq_kv_cache(C.Structure):
    _fields_ = [("d_words", C.c_void_p), ("cap_words", C.c_uint64), ("d_offsets", C.c_void_p),
                ("offsets_cap", C.c_uint64), ("d_table", C.c_void_p), ("table_cap", C.c_uint64),
                ("d_tail", C.c_void_p), ("d_stats", C.c_void_p), ("heads", C.c_int32), ("head_dim", C.c_int32),
                ("params", hq_params), ("tokens", C.c_int64), ("chunks", C.c_uint64), ("appends", C.c_uint64)]


class hq_calib_spec(C.Structure):
    _fields_ = [("target_bps", C.c_double), ("tol", C.c_double), ("alpha_lo", C.c_double), ("alpha_hi", C.c_double),
                ("k_lo", C.c_int32), ("k_hi", C.c_int32), ("max_iter", C.c_int32), ("reserved", C.c_int32)]


class hq_calib_result(C.Structure):
    _fields_ = [("alpha", C.c_float), ("k", C.c_int32), ("bps", C.c_double), ("evaluations", C.c_int32),
                ("status", C.c_uint32)]


STATS_BYTES = 40
assert C.sizeof(hq_calib_spec) == 48 and C.sizeof(hq_calib_result) == 24
assert C.sizeof(hq_params) == 48 and C.sizeof(hq_stats) == STATS_BYTES and C.sizeof(hq_kv_append_row) == 32
assert C.sizeof(hq_kv_cache) == 144

# C entry points: name -> (restype, argtypes)
EXPORTS = {
    "hq_stream_bound": (C.c_int, [C.c_int64, C.c_int64, C.POINTER(hq_params), C.c_uint32, C.POINTER(C.c_uint64),
                                  C.POINTER(C.c_uint64)]),
    "hq_workspace_bytes": (C.c_int, [C.c_uint64, C.POINTER(C.c_size_t)]),
    "hq_quantize": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.POINTER(hq_params), C.c_void_p,
                              C.c_uint64, C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "hq_dequantize": (C.c_int, [C.c_void_p, C.c_uint64, C.c_void_p, C.c_int64, C.c_int64, C.POINTER(hq_params),
                                C.c_void_p, C.c_int, C.c_int64, C.c_void_p, C.c_void_p]),
    "hq_rate": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.POINTER(hq_params), C.c_void_p, C.c_void_p]),
    "hq_rate_kv": (C.c_int, [C.c_void_p, C.c_int32, C.c_int64, C.c_int64, C.c_int64, C.c_int64, C.POINTER(hq_params),
                             C.c_void_p, C.c_void_p]),
    "hq_calibrate": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.POINTER(hq_params),
                               C.POINTER(hq_calib_spec), C.c_void_p, C.c_void_p, C.POINTER(hq_calib_result)]),
    "hq_calibrate_kv": (C.c_int, [C.c_void_p, C.c_int32, C.c_int64, C.c_int64, C.c_int64, C.c_int64,
                                  C.POINTER(hq_params), C.POINTER(hq_calib_spec), C.c_void_p, C.c_void_p,
                                  C.POINTER(hq_calib_result)]),
    "hq_gemv_workspace_bytes": (C.c_int, [C.c_int64, C.c_int64, C.POINTER(C.c_size_t)]),
    "hq_gemv": (C.c_int, [C.c_void_p, C.c_uint64, C.c_void_p, C.c_int64, C.c_int64, C.POINTER(hq_params),
                          C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p, C.c_void_p]),
    "hq_kv_scores": (C.c_int, [C.POINTER(hq_kv_cache), C.c_void_p, C.c_int32, C.c_void_p, C.c_int64, C.c_int64,
                               C.c_void_p]),
    "hq_debug_set_encode_path": (C.c_int, [C.c_int]),
    "hq_debug_nearest": (C.c_int, [C.c_int, C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p]),
    "hq_kv_init": (C.c_int, [C.POINTER(hq_kv_cache), C.c_int32, C.c_int32, C.POINTER(hq_params), C.c_void_p,
                             C.c_uint64, C.c_void_p, C.c_uint64, C.c_void_p, C.c_uint64, C.c_void_p, C.c_void_p,
                             C.c_void_p]),
    "hq_kv_append": (C.c_int, [C.POINTER(hq_kv_cache), C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.c_float,
                               C.c_void_p, C.c_size_t, C.c_void_p]),
    "hq_kv_read": (C.c_int, [C.POINTER(hq_kv_cache), C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_int64,
                             C.c_void_p]),
    "hq_status_string": (C.c_char_p, [C.c_int]),
    "hq_device_check": (C.c_int, []),
    "hq_debug_set_spin_limit": (None, [C.c_uint32]),
    "hq_quantize_static": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.POINTER(hq_params), C.c_void_p,
                                     C.c_uint64, C.c_void_p, C.c_void_p, C.c_void_p]),
    "hq_haar_rotation": (C.c_int, [C.c_uint64, C.c_void_p, C.c_void_p]),
    "hq_offsets_add": (C.c_int, [C.c_void_p, C.c_uint64, C.c_uint64, C.c_void_p]),
    "hq_batch_workspace_bytes": (C.c_int, [C.c_int64, C.c_uint64, C.POINTER(C.c_size_t)]),
    "hq_quantize_batch": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.c_int64, C.c_int64,
                                    C.POINTER(hq_params), C.c_void_p, C.c_uint64, C.c_uint64, C.c_void_p, C.c_void_p,
                                    C.c_void_p, C.c_size_t, C.c_void_p]),
    "hq_dequantize_batch": (C.c_int, [C.c_void_p, C.c_uint64, C.c_uint64, C.c_void_p, C.c_int64, C.c_int64,
                                      C.c_int64, C.POINTER(hq_params), C.c_void_p, C.c_int, C.c_int64, C.c_int64,
                                      C.c_void_p, C.c_void_p]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m lattice_entropy_coded_b200.build`")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in EXPORTS.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


class HQError(RuntimeError):
    pass


def _check(rc: int, what: str) -> int:
    if rc < 0:
        raise HQError(f"{what}: {hq_status_string(rc)} ({rc})")
    return rc


def _ptr(t) -> int | None:
    if t is None:
        return None
    assert isinstance(t, torch.Tensor)
    return t.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, torch.cuda.Stream):
        return s.cuda_stream
    return int(s)


def make_params(lattice="E8", alpha=1.0, rice_k=2, seed=0, dither=0, rotation: torch.Tensor | None = None,
                dk_last: int = 0) -> hq_params:
    """rotation: a KV cache's dense rotation (fp32 [128, 128] on the device, e.g. from
    hq_haar_rotation), or None for the sign diagonal and H_128.  The params hold only its
    address: the caller keeps the tensor alive and unchanged.  dk_last: the last symbol of
    each A2 / D4 / E8 block is Rice coded with max(rice_k - dk_last, 0) (0: one parameter)."""
    lat = LATTICES[lattice] if isinstance(lattice, str) else int(lattice)
    rot = None
    if rotation is not None:
        assert rotation.dtype == torch.float32 and rotation.is_contiguous() and tuple(rotation.shape) == (128, 128)
        rot = rotation.data_ptr()
    return hq_params(128, lat, float(alpha), int(rice_k), int(seed) & (2**64 - 1), int(dither), 32, rot,
                     int(dk_last), 0)


# ------------------------------------------------------------------ C entry points
def hq_status_string(code: int) -> str:
    return _lib.hq_status_string(int(code)).decode()


def hq_device_check() -> int:
    return int(_lib.hq_device_check())


def hq_debug_set_spin_limit(polls: int) -> None:
    _lib.hq_debug_set_spin_limit(int(polls))


def hq_gemv_workspace_bytes(rows: int, cols: int) -> int:
    b = C.c_size_t()
    _check(_lib.hq_gemv_workspace_bytes(rows, cols, C.byref(b)), "hq_gemv_workspace_bytes")
    return int(b.value)


def hq_gemv(stream: torch.Tensor, stream_words: int, offsets: torch.Tensor, rows: int, cols: int, params: hq_params,
            x: torch.Tensor, y: torch.Tensor, workspace: torch.Tensor, stats: torch.Tensor | None = None,
            cuda_stream=None) -> int:
    """y (fp32 [rows]) = W x for the compressed W; x bf16 [cols]."""
    assert x.dtype == torch.bfloat16 and x.is_contiguous() and y.dtype == torch.float32
    return _check(_lib.hq_gemv(_ptr(stream), stream_words, _ptr(offsets), rows, cols, C.byref(params), _ptr(x),
                               _ptr(y), _ptr(workspace), workspace.numel(), _ptr(stats), _stream(cuda_stream)),
                  "hq_gemv")


def hq_kv_scores(cache: hq_kv_cache, q: torch.Tensor, group: int, scores: torch.Tensor, length: int,
                 cuda_stream=None) -> int:
    """q bf16 [heads * group, 128]; scores fp32 [heads * group, >= length]."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous() and scores.dtype == torch.float32
    return _check(_lib.hq_kv_scores(C.byref(cache), _ptr(q), group, _ptr(scores), length, scores.stride(0),
                                    _stream(cuda_stream)), "hq_kv_scores")


def hq_rate(x: torch.Tensor, params: hq_params, stats: torch.Tensor, cuda_stream=None, ld: int | None = None) -> int:
    """Rate of hq_quantize(x, params) without its stream, into stats (payload_bits, stream_words, ...)."""
    rows, cols = x.shape
    ld = x.stride(0) if ld is None else ld
    return _check(_lib.hq_rate(_ptr(x), rows, cols, ld, C.byref(params), _ptr(stats), _stream(cuda_stream)), "hq_rate")


def hq_rate_kv(kv: torch.Tensor, params: hq_params, stats: torch.Tensor, tok0: int = 0, cuda_stream=None) -> int:
    """kv: bf16 [heads, T, 128], unit stride in the last dimension; tokens at positions tok0..tok0+T-1."""
    H, T, D = kv.shape
    assert D == 128 and kv.stride(2) == 1
    return _check(_lib.hq_rate_kv(_ptr(kv), H, T, kv.stride(1), kv.stride(0), tok0, C.byref(params), _ptr(stats),
                                  _stream(cuda_stream)), "hq_rate_kv")


def calib_spec(target_bps: float, tol: float = 0.002, k_lo: int = 0, k_hi: int = 6, alpha_lo: float = 1e-3,
               alpha_hi: float = 1e4, max_iter: int = 60) -> hq_calib_spec:
    return hq_calib_spec(float(target_bps), float(tol), float(alpha_lo), float(alpha_hi), int(k_lo), int(k_hi),
                         int(max_iter), 0)


def _calib_result(r: hq_calib_result) -> dict:
    return {"alpha": float(r.alpha), "k": int(r.k), "bps": float(r.bps), "evaluations": int(r.evaluations),
            "status": int(r.status)}


def hq_calibrate(x: torch.Tensor, params: hq_params, spec: hq_calib_spec, stats: torch.Tensor, cuda_stream=None,
                 ld: int | None = None) -> dict:
    """Synchronous: alpha (and k) for spec.target_bps on the device; see hq.h."""
    rows, cols = x.shape
    ld = x.stride(0) if ld is None else ld
    out = hq_calib_result()
    _check(_lib.hq_calibrate(_ptr(x), rows, cols, ld, C.byref(params), C.byref(spec), _ptr(stats),
                             _stream(cuda_stream), C.byref(out)), "hq_calibrate")
    return _calib_result(out)


def hq_calibrate_kv(kv: torch.Tensor, params: hq_params, spec: hq_calib_spec, stats: torch.Tensor, tok0: int = 0,
                    cuda_stream=None) -> dict:
    H, T, D = kv.shape
    assert D == 128 and kv.stride(2) == 1
    out = hq_calib_result()
    _check(_lib.hq_calibrate_kv(_ptr(kv), H, T, kv.stride(1), kv.stride(0), tok0, C.byref(params), C.byref(spec),
                                _ptr(stats), _stream(cuda_stream), C.byref(out)), "hq_calibrate_kv")
    return _calib_result(out)


def hq_haar_rotation(seed: int, out: torch.Tensor | None = None, cuda_stream=None) -> torch.Tensor:
    """A Haar-uniform 128 x 128 orthogonal fp32 matrix drawn on the device for this seed."""
    if out is None:
        out = torch.empty(128, 128, dtype=torch.float32, device="cuda")
    assert out.dtype == torch.float32 and out.is_contiguous() and tuple(out.shape) == (128, 128)
    _check(_lib.hq_haar_rotation(int(seed) & (2**64 - 1), _ptr(out), _stream(cuda_stream)), "hq_haar_rotation")
    return out


def hq_offsets_add(offsets: torch.Tensor, base: int, cuda_stream=None) -> int:
    """offsets (int64 / uint64 words of a stream's chunk offsets, on the device) += base, in place."""
    assert offsets.dtype == torch.int64 and offsets.is_contiguous()
    return _check(_lib.hq_offsets_add(_ptr(offsets), offsets.numel(), int(base), _stream(cuda_stream)),
                  "hq_offsets_add")


def hq_debug_set_encode_path(path: int) -> int:
    """0 = by size, 1 = per-warp, 2 = grouped, 3 = wide, 4 = single-CTA encoder (testing aid)."""
    return _check(_lib.hq_debug_set_encode_path(int(path)), "hq_debug_set_encode_path")


def hq_debug_nearest(lattice, v: torch.Tensor, q: torch.Tensor, cuda_stream=None) -> int:
    """v: fp32 [n, dim] on the device; q: int32 [n, dim] (codes out)."""
    lat = LATTICES[lattice] if isinstance(lattice, str) else int(lattice)
    assert v.dtype == torch.float32 and q.dtype == torch.int32 and v.is_contiguous() and q.is_contiguous()
    assert v.shape == q.shape and v.dim() == 2
    return _check(_lib.hq_debug_nearest(lat, _ptr(v), v.shape[0], _ptr(q), _stream(cuda_stream)), "hq_debug_nearest")


def hq_stream_bound(rows: int, cols: int, params: hq_params, max_abs_symbol: int = 0):
    w, n = C.c_uint64(), C.c_uint64()
    _check(_lib.hq_stream_bound(rows, cols, C.byref(params), max_abs_symbol, C.byref(w), C.byref(n)),
           "hq_stream_bound")
    return int(w.value), int(n.value)


def hq_workspace_bytes(n_chunks: int) -> int:
    b = C.c_size_t()
    _check(_lib.hq_workspace_bytes(n_chunks, C.byref(b)), "hq_workspace_bytes")
    return int(b.value)


def hq_quantize(x: torch.Tensor, params: hq_params, stream: torch.Tensor, offsets: torch.Tensor,
                stats: torch.Tensor | None, workspace: torch.Tensor, cuda_stream=None, ld: int | None = None) -> int:
    """x: bf16 [rows, cols] (row stride ld, default x.stride(0)); stream: int32/uint32 words;
    offsets: int64 [n_chunks + 1]; stats: uint8 [STATS_BYTES] or None; workspace: uint8."""
    rows, cols = x.shape
    ld = x.stride(0) if ld is None else ld
    return _check(_lib.hq_quantize(_ptr(x), rows, cols, ld, C.byref(params), _ptr(stream), stream.numel(),
                                   _ptr(offsets), _ptr(stats), _ptr(workspace), workspace.numel(),
                                   _stream(cuda_stream)), "hq_quantize")


def hq_batch_workspace_bytes(batch: int, n_chunks: int) -> int:
    b = C.c_size_t()
    _check(_lib.hq_batch_workspace_bytes(batch, n_chunks, C.byref(b)), "hq_batch_workspace_bytes")
    return int(b.value)


def hq_quantize_batch(x: torch.Tensor, params: hq_params, stream: torch.Tensor, offsets: torch.Tensor,
                      stats: torch.Tensor | None, workspace: torch.Tensor, cap_words: int | None = None,
                      cuda_stream=None) -> int:
    """x: bf16 [batch, rows, cols] (row stride x.stride(1), item stride x.stride(0));
    stream: int32 [batch, S] words (item i's stream is row i, cap_words <= S words);
    offsets: int64 [batch, n_chunks + 1]; stats: uint8 [batch, STATS_BYTES] or None."""
    B, rows, cols = x.shape
    assert stream.dim() == 2 and stream.shape[0] == B and stream.stride(1) == 1
    cap = stream.shape[1] if cap_words is None else cap_words
    return _check(_lib.hq_quantize_batch(_ptr(x), B, x.stride(0), rows, cols, x.stride(1), C.byref(params),
                                         _ptr(stream), stream.stride(0), cap, _ptr(offsets), _ptr(stats),
                                         _ptr(workspace), workspace.numel(), _stream(cuda_stream)),
                  "hq_quantize_batch")


def hq_dequantize_batch(stream: torch.Tensor, stream_words: int, offsets: torch.Tensor, rows: int, cols: int,
                        params: hq_params, out: torch.Tensor, stats: torch.Tensor | None = None,
                        cuda_stream=None) -> int:
    """stream: int32 [batch, S]; offsets: int64 [batch, n_chunks + 1]; out: bf16 or fp32
    [batch, rows, cols] (row stride out.stride(1), item stride out.stride(0))."""
    B = out.shape[0]
    assert out.dtype in (torch.float32, torch.bfloat16)
    dt = 1 if out.dtype == torch.float32 else 0
    return _check(_lib.hq_dequantize_batch(_ptr(stream), stream.stride(0), stream_words, _ptr(offsets), B, rows,
                                           cols, C.byref(params), _ptr(out), dt, out.stride(1), out.stride(0),
                                           _ptr(stats), _stream(cuda_stream)), "hq_dequantize_batch")


def hq_quantize_static(x: torch.Tensor, params: hq_params, stream: torch.Tensor, offsets: torch.Tensor,
                       stats: torch.Tensor | None, cuda_stream=None, ld: int | None = None) -> int:
    """hq_quantize for callers that cannot allocate: its scratch is a fixed array inside
    libhq.so (limit HQ_STATIC_MAX_CHUNKS chunks; overlapping calls on the GPU race)."""
    rows, cols = x.shape
    ld = x.stride(0) if ld is None else ld
    return _check(_lib.hq_quantize_static(_ptr(x), rows, cols, ld, C.byref(params), _ptr(stream), stream.numel(),
                                          _ptr(offsets), _ptr(stats), _stream(cuda_stream)), "hq_quantize_static")


def hq_dequantize(stream: torch.Tensor, stream_words: int, offsets: torch.Tensor, rows: int, cols: int,
                  params: hq_params, out: torch.Tensor, stats: torch.Tensor | None = None, cuda_stream=None) -> int:
    """out: bf16 or fp32 [rows, cols] (row stride out.stride(0))."""
    dt = 1 if out.dtype == torch.float32 else 0
    assert out.dtype in (torch.float32, torch.bfloat16)
    return _check(_lib.hq_dequantize(_ptr(stream), stream_words, _ptr(offsets), rows, cols, C.byref(params),
                                     _ptr(out), dt, out.stride(0), _ptr(stats), _stream(cuda_stream)),
                  "hq_dequantize")


def hq_kv_init(cache: hq_kv_cache, heads: int, head_dim: int, params: hq_params, words: torch.Tensor,
               offsets: torch.Tensor, table: torch.Tensor, tail: torch.Tensor, stats: torch.Tensor,
               cuda_stream=None) -> int:
    return _check(_lib.hq_kv_init(C.byref(cache), heads, head_dim, C.byref(params), _ptr(words), words.numel(),
                                  _ptr(offsets), offsets.numel(), _ptr(table), table.numel() // 32, _ptr(tail),
                                  _ptr(stats), _stream(cuda_stream)), "hq_kv_init")


def hq_kv_append(cache: hq_kv_cache, kv: torch.Tensor, alpha: float, workspace: torch.Tensor,
                 cuda_stream=None) -> int:
    """kv: bf16 [heads, T, 128] with unit stride in the last dimension."""
    H, T, D = kv.shape
    assert D == 128 and kv.stride(2) == 1
    return _check(_lib.hq_kv_append(C.byref(cache), _ptr(kv), T, kv.stride(1), kv.stride(0), float(alpha),
                                    _ptr(workspace), workspace.numel(), _stream(cuda_stream)), "hq_kv_append")


def hq_kv_read(cache: hq_kv_cache, out: torch.Tensor, length: int, cuda_stream=None) -> int:
    """out: bf16 or fp32 [heads, >= length, 128]."""
    dt = 1 if out.dtype == torch.float32 else 0
    return _check(_lib.hq_kv_read(C.byref(cache), _ptr(out), dt, length, out.stride(1), out.stride(0),
                                  _stream(cuda_stream)), "hq_kv_read")


# ------------------------------------------------------------------ torch-allocated wrappers
def stats_tensor(device="cuda") -> torch.Tensor:
    return torch.zeros(STATS_BYTES, dtype=torch.uint8, device=device)


def read_stats(t: torch.Tensor) -> dict:
    b = bytes(t.cpu().numpy().tobytes())
    s = hq_stats.from_buffer_copy(b)
    return {"status": s.status, "max_symbol": s.max_symbol, "payload_bits": s.payload_bits,
            "stream_words": s.stream_words, "max_abs_code": s.max_abs_code,
            "int8_overflow_count": s.int8_overflow_count}


@dataclass
class Compressed:
    """A quantized matrix: its stream words, chunk offsets and the parameters."""
    words: torch.Tensor      # int32, >= n_words
    offsets: torch.Tensor    # int64 [n_chunks + 1]
    rows: int
    cols: int
    params: hq_params
    stats: torch.Tensor      # uint8 [STATS_BYTES] hq_stats


class Codec:
    """Owns the device buffers of repeated quantize / dequantize calls of one shape."""

    def __init__(self, rows: int, cols: int, params: hq_params, max_abs_symbol: int = 0, device="cuda",
                 cap_words: int | None = None):
        self.rows, self.cols, self.params = rows, cols, params
        bound, self.n_chunks = hq_stream_bound(rows, cols, params, max_abs_symbol)
        self.cap_words = bound if cap_words is None else cap_words
        self.words = torch.empty(max(self.cap_words, 1), dtype=torch.int32, device=device)
        self.offsets = torch.empty(self.n_chunks + 1, dtype=torch.int64, device=device)
        self.stats = stats_tensor(device)
        self.workspace = torch.empty(hq_workspace_bytes(self.n_chunks), dtype=torch.uint8, device=device)

    def quantize(self, x: torch.Tensor, cuda_stream=None) -> Compressed:
        hq_quantize(x, self.params, self.words[:self.cap_words], self.offsets, self.stats, self.workspace,
                    cuda_stream)
        return Compressed(self.words, self.offsets, self.rows, self.cols, self.params, self.stats)

    def dequantize(self, c: Compressed, out: torch.Tensor, stats: torch.Tensor | None = None,
                   cuda_stream=None) -> torch.Tensor:
        hq_dequantize(c.words, self.cap_words, c.offsets, c.rows, c.cols, c.params, out, stats, cuda_stream)
        return out

    def gemv(self, c: Compressed, x: torch.Tensor, y: torch.Tensor, stats: torch.Tensor | None = None,
             cuda_stream=None) -> torch.Tensor:
        """y = W x straight from the compressed W (no bf16 copy of W is made)."""
        if getattr(self, "_gemv_ws", None) is None:
            self._gemv_ws = torch.empty(hq_gemv_workspace_bytes(self.rows, self.cols), dtype=torch.uint8,
                                        device=self.words.device)
        hq_gemv(c.words, self.cap_words, c.offsets, c.rows, c.cols, c.params, x, y, self._gemv_ws, stats, cuda_stream)
        return y


class KVCache:
    """A compressed K or V cache (one layer) with torch-allocated device buffers.
    rotation: a dense rotation for this cache (fp32 [128, 128], e.g. hq_haar_rotation(seed)),
    used in place of the sign diagonal and H_128; the cache keeps a reference to it."""

    def __init__(self, heads: int, max_tokens: int, params: hq_params, bits_per_scalar: float = 4.0,
                 max_appends: int = 4096, max_append_tokens: int = 4096, device="cuda",
                 rotation: torch.Tensor | None = None):
        if rotation is not None:
            assert rotation.dtype == torch.float32 and rotation.is_contiguous() and tuple(rotation.shape) == (128, 128)
            params = hq_params.from_buffer_copy(bytes(params))
            params.rotation = rotation.data_ptr()
        self.rotation = rotation
        max_chunks = heads * ((max_tokens + 31) // 32 + max_appends)
        cap = int(heads * max_tokens * 128 * bits_per_scalar / 32) + max_chunks * 64 + 1024
        self.words = torch.empty(cap, dtype=torch.int32, device=device)
        self.offsets = torch.empty(max_chunks + 1, dtype=torch.int64, device=device)
        self.table = torch.zeros(max_appends * 32, dtype=torch.uint8, device=device)
        self.tail = torch.zeros(2, dtype=torch.int64, device=device)
        self.stats = stats_tensor(device)
        self.workspace = torch.empty(hq_workspace_bytes(heads * ((max_append_tokens + 31) // 32)),
                                     dtype=torch.uint8, device=device)
        self.heads = heads
        self.cache = hq_kv_cache()
        hq_kv_init(self.cache, heads, 128, params, self.words, self.offsets, self.table, self.tail, self.stats)

    @property
    def tokens(self) -> int:
        return int(self.cache.tokens)

    def append(self, kv: torch.Tensor, alpha: float, cuda_stream=None):
        hq_kv_append(self.cache, kv, alpha, self.workspace, cuda_stream)

    def read(self, out: torch.Tensor, length: int | None = None, cuda_stream=None) -> torch.Tensor:
        hq_kv_read(self.cache, out, self.tokens if length is None else length, cuda_stream)
        return out

    def scores(self, q: torch.Tensor, group: int, out: torch.Tensor, length: int | None = None,
               cuda_stream=None) -> torch.Tensor:
        """out[h * group + g, t] = K[h, t] . q[h * group + g] straight from the compressed cache."""
        hq_kv_scores(self.cache, q, group, out, self.tokens if length is None else length, cuda_stream)
        return out
