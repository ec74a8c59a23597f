"""Plain CPU oracle of the HyperQuant quantize / dequantize path (test infrastructure).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this package.  The product library
(``lattice_entropy_coded_b200``) never imports it and shares no code with it.

The arithmetic lives in ``hqref.c`` (plain C99, strict IEEE fp32, no FMA
contraction); this module compiles it with gcc on first use and marshals numpy
arrays through ctypes.  Every function here is argument marshalling only.
"""
from __future__ import annotations

import contextlib
import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hqref.c")
_HDR = os.path.join(_HERE, "hqref.h")
_LIB = os.path.join(_HERE, "libhqref.so")
CFLAGS = ["-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fno-builtin", "-shared", "-fPIC"]

Z, A2, D4, E8 = 0, 1, 2, 3
LATTICES = {"Z": Z, "A2": A2, "D4": D4, "E8": E8}
DIM = {Z: 1, A2: 2, D4: 4, E8: 8}

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile hqref.c into libhqref.so (gcc, strict fp32); returns the path."""
    stale = (not os.path.exists(_LIB)) or any(
        os.path.getmtime(p) > os.path.getmtime(_LIB) for p in (_SRC, _HDR))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(C.CDLL(build()))
    return _lib


@contextlib.contextmanager
def using_library(path: str):
    """Temporarily route every oracle call through another build of hqref.c
    (used by the tests that plant a mistake in a copy of the oracle)."""
    global _lib
    lib()
    old = _lib
    _lib = _bind(C.CDLL(path))
    try:
        yield
    finally:
        _lib = old


def build_variant(src_text: str, out_path: str) -> str:
    """Compile a modified copy of hqref.c (same flags) to out_path."""
    d = os.path.dirname(out_path)
    src = os.path.join(d, "hqref_variant.c")
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", *CFLAGS, "-I", _HERE, "-o", out_path, src, "-lm"], check=True)
    return out_path


def source() -> str:
    with open(_SRC) as f:
        return f.read()


_p = C.c_void_p
_i32, _i64, _u32, _u64, _f32 = C.c_int, C.c_int64, C.c_uint32, C.c_uint64, C.c_float


def _bind(L):
    sig = {
        "hqref_splitmix64": (_u64, [_u64, _u64]),
        "hqref_sign": (_i32, [_u64, _u64]),
        "hqref_bf16_to_f32": (_f32, [C.c_uint16]),
        "hqref_f32_to_bf16": (C.c_uint16, [_f32]),
        "hqref_fwht128": (None, [_p]),
        "hqref_scale_fwd": (_f32, [_f32]),
        "hqref_scale_inv": (_f32, [_f32]),
        "hqref_lattice_dim": (_i32, [_i32]),
        "hqref_decode": (None, [_i32, _p, _p]),
        "hqref_decode_many": (None, [_i32, _p, C.c_int64, _p]),
        "hqref_point": (None, [_i32, _p, _p]),
        "hqref_is_member": (_i32, [_i32, _p]),
        "hqref_dither_uniform": (_f32, [_u64, _u64]),
        "hqref_dither_block": (None, [_i32, _u64, _u64, _p]),
        "hqref_strip": (None, [_i32, _p, _p, _p]),
        "hqref_reinsert": (None, [_i32, _p, _u32, _p]),
        "hqref_zigzag": (_u32, [C.c_int32]),
        "hqref_unzigzag": (C.c_int32, [_u32]),
        "hqref_rice_concat": (_u64, [_p, _i64, _i32, _p, _u64]),
        "hqref_rice_concat_decode": (_i32, [_p, _u64, _i64, _i32, _p]),
        "hqref_encode_chunk": (_u64, [_i32, _i32, _p, _i32, _p, _u64, _p, _i32]),
        "hqref_decode_chunk": (_i32, [_i32, _i32, _p, _u64, _i32, _p, _i32]),
        "hqref_symbol_k": (_i32, [_i32, _i32, _i32, _i32]),
        "hqref_rice_concat_k": (_u64, [_p, _i64, _p, _p, _u64]),
        "hqref_quantize_tile": (None, [_p, _i32, _f32, _u64, _u64, _i32, _u64, _p]),
        "hqref_dequantize_tile": (None, [_p, _i32, _f32, _u64, _u64, _i32, _u64, _p]),
        "hqref_n_chunks": (_i64, [_i64, _i64]),
        "hqref_quantize": (_i64, [_p, _i64, _i64, _i64, _i32, _f32, _i32, _u64, _i32, _i64, _i64, _p, _u64,
                                  _p, _p, _i32]),
        "hqref_dequantize": (_i32, [_p, _p, _i64, _i64, _i32, _f32, _i32, _u64, _i32, _i64, _i64, _i32, _p,
                                    _i64, _i32]),
        "hqref_kv_append": (_i64, [_p, _i64, _i64, _i64, _i64, _i64, _i32, _f32, _i32, _u64, _i32, _p, _u64,
                                   _u64, _p, _p, _p, _i32]),
        "hqref_kv_read_append": (_i32, [_p, _p, _i64, _i64, _i64, _i32, _f32, _i32, _u64, _i32, _i32, _p,
                                        _i64, _i64, _i64, _p, _i32]),
        "hqref_rotate_fwd": (None, [_p, _p, _p]),
        "hqref_rotate_inv": (None, [_p, _p, _p]),
        "hqref_scale_inv_rot": (_f32, [_f32]),
        "hqref_quantize_tile_rot": (None, [_p, _i32, _f32, _p, _u64, _i32, _u64, _p]),
        "hqref_dequantize_tile_rot": (None, [_p, _i32, _f32, _p, _u64, _i32, _u64, _p]),
        "hqref_rot_gaussian": (C.c_double, [_u64, _u64]),
        "hqref_code_range": (None, [_p, _i64, _p, _p]),
        "hqref_quantize_range": (None, [_p, _i64, _i64, _i64, _i32, _f32, _u64, _i32, _i64, _i64, _p, _p]),
        "hqref_kv_range": (None, [_p, _i64, _i64, _i64, _i64, _i64, _i32, _f32, _u64, _i32, _p, _p, _p]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"] or a.ndim == 0
    return a.ctypes.data_as(C.c_void_p)


def _as_u16(x) -> np.ndarray:
    """bf16 data as a uint16 numpy array (accepts a torch bf16 tensor or uint16 array)."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


# ---------------------------------------------------------------- scalar pieces
def splitmix64(s: int, i: int) -> int:
    return int(lib().hqref_splitmix64(s & (2**64 - 1), i & (2**64 - 1)))


def sign(seed: int, j: int) -> int:
    return int(lib().hqref_sign(seed, j))


def bf16_to_f32(b: int) -> float:
    return float(lib().hqref_bf16_to_f32(b))


def f32_to_bf16(f: float) -> int:
    return int(lib().hqref_f32_to_bf16(f))


def fwht128(v) -> np.ndarray:
    a = np.array(v, dtype=np.float32).copy()
    assert a.shape == (128,)
    lib().hqref_fwht128(_ptr(a))
    return a


def scale_fwd(alpha: float) -> float:
    return float(lib().hqref_scale_fwd(alpha))


def scale_inv(alpha: float) -> float:
    return float(lib().hqref_scale_inv(alpha))


def decode(lat: int, v) -> np.ndarray:
    a = np.ascontiguousarray(v, dtype=np.float32)
    assert a.shape == (DIM[lat],)
    q = np.zeros(DIM[lat], dtype=np.int32)
    lib().hqref_decode(lat, _ptr(a), _ptr(q))
    return q


def decode_many(lat: int, v) -> np.ndarray:
    """hqref_decode on every row of v [n, dim]."""
    a = np.ascontiguousarray(v, dtype=np.float32)
    assert a.ndim == 2 and a.shape[1] == DIM[lat]
    q = np.zeros(a.shape, dtype=np.int32)
    lib().hqref_decode_many(lat, _ptr(a), a.shape[0], _ptr(q))
    return q


def point(lat: int, q) -> np.ndarray:
    a = np.ascontiguousarray(q, dtype=np.int32)
    p = np.zeros(DIM[lat], dtype=np.float32)
    lib().hqref_point(lat, _ptr(a), _ptr(p))
    return p


def is_member(lat: int, q) -> bool:
    a = np.ascontiguousarray(q, dtype=np.int32)
    return bool(lib().hqref_is_member(lat, _ptr(a)))


def dither_uniform(seed: int, e: int) -> float:
    return float(lib().hqref_dither_uniform(seed, e))


def dither_block(lat: int, seed: int, e0: int) -> np.ndarray:
    d = np.zeros(DIM[lat], dtype=np.float32)
    lib().hqref_dither_block(lat, seed, e0, _ptr(d))
    return d


def strip(lat: int, q):
    a = np.ascontiguousarray(q, dtype=np.int32)
    m = np.zeros(DIM[lat], dtype=np.int32)
    c = np.zeros(1, dtype=np.uint32)
    lib().hqref_strip(lat, _ptr(a), _ptr(m), _ptr(c))
    return m, int(c[0])


def reinsert(lat: int, m, coset: int) -> np.ndarray:
    a = np.ascontiguousarray(m, dtype=np.int32)
    q = np.zeros(DIM[lat], dtype=np.int32)
    lib().hqref_reinsert(lat, _ptr(a), coset, _ptr(q))
    return q


def zigzag(m: int) -> int:
    return int(lib().hqref_zigzag(m))


def unzigzag(z: int) -> int:
    return int(lib().hqref_unzigzag(z))


def rice_concat(z, k: int):
    zz = np.ascontiguousarray(z, dtype=np.uint32)
    nbits = int(lib().hqref_rice_concat(_ptr(zz), zz.size, k, None, 0))
    out = np.zeros((nbits + 31) // 32, dtype=np.uint32)
    lib().hqref_rice_concat(_ptr(zz), zz.size, k, _ptr(out), out.size)
    return out, nbits


def rice_concat_decode(words, nbits: int, n: int, k: int) -> np.ndarray:
    w = np.ascontiguousarray(words, dtype=np.uint32)
    z = np.zeros(n, dtype=np.uint32)
    rc = lib().hqref_rice_concat_decode(_ptr(w), nbits, n, k, _ptr(z))
    if rc != 0:
        raise ValueError("corrupt Rice stream")
    return z


def symbol_k(lat: int, k: int, dk_last: int, i: int) -> int:
    return int(lib().hqref_symbol_k(lat, k, dk_last, i))


def rice_concat_k(z, ks):
    zz = np.ascontiguousarray(z, dtype=np.uint32)
    kk = np.ascontiguousarray(ks, dtype=np.int32)
    assert kk.size == zz.size
    nbits = int(lib().hqref_rice_concat_k(_ptr(zz), zz.size, _ptr(kk), None, 0))
    out = np.zeros((nbits + 31) // 32, dtype=np.uint32)
    lib().hqref_rice_concat_k(_ptr(zz), zz.size, _ptr(kk), _ptr(out), out.size)
    return out, nbits


def encode_chunk(lat: int, k: int, codes, dk_last: int = 0):
    q = np.ascontiguousarray(codes, dtype=np.int32)
    assert q.size % 128 == 0
    nt = q.size // 128
    pb = np.zeros(1, dtype=np.uint64)
    n = int(lib().hqref_encode_chunk(lat, k, _ptr(q), nt, None, 0, _ptr(pb), dk_last))
    out = np.zeros(n, dtype=np.uint32)
    lib().hqref_encode_chunk(lat, k, _ptr(q), nt, _ptr(out), n, _ptr(pb), dk_last)
    return out, int(pb[0])


def decode_chunk(lat: int, k: int, words, ntiles: int, dk_last: int = 0) -> np.ndarray:
    w = np.ascontiguousarray(words, dtype=np.uint32)
    q = np.zeros(ntiles * 128, dtype=np.int32)
    if lib().hqref_decode_chunk(lat, k, _ptr(w), w.size, ntiles, _ptr(q), dk_last) != 0:
        raise ValueError("corrupt chunk")
    return q


def quantize_tile(x_u16, lat, alpha, seed, sign_col0=0, dither=0, e0=0) -> np.ndarray:
    x = np.ascontiguousarray(x_u16, dtype=np.uint16)
    q = np.zeros(128, dtype=np.int32)
    lib().hqref_quantize_tile(_ptr(x), lat, alpha, seed, sign_col0, dither, e0, _ptr(q))
    return q


def dequantize_tile(q, lat, alpha, seed, sign_col0=0, dither=0, e0=0) -> np.ndarray:
    a = np.ascontiguousarray(q, dtype=np.int32)
    out = np.zeros(128, dtype=np.float32)
    lib().hqref_dequantize_tile(_ptr(a), lat, alpha, seed, sign_col0, dither, e0, _ptr(out))
    return out


def rotate_fwd(Q, x) -> np.ndarray:
    q = np.ascontiguousarray(Q, dtype=np.float32)
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(128, dtype=np.float32)
    lib().hqref_rotate_fwd(_ptr(q), _ptr(a), _ptr(out))
    return out


def rotate_inv(Q, z) -> np.ndarray:
    q = np.ascontiguousarray(Q, dtype=np.float32)
    a = np.ascontiguousarray(z, dtype=np.float32)
    out = np.zeros(128, dtype=np.float32)
    lib().hqref_rotate_inv(_ptr(q), _ptr(a), _ptr(out))
    return out


def scale_inv_rot(alpha: float) -> float:
    return float(lib().hqref_scale_inv_rot(alpha))


def quantize_tile_rot(x_u16, lat, alpha, Q, seed, dither=0, e0=0) -> np.ndarray:
    x = np.ascontiguousarray(x_u16, dtype=np.uint16)
    r_keep, rp = _rot_ptr(Q)
    q = np.zeros(128, dtype=np.int32)
    lib().hqref_quantize_tile_rot(_ptr(x), lat, alpha, rp, seed, dither, e0, _ptr(q))
    return q


def dequantize_tile_rot(q, lat, alpha, Q, seed, dither=0, e0=0) -> np.ndarray:
    a = np.ascontiguousarray(q, dtype=np.int32)
    r_keep, rp = _rot_ptr(Q)
    out = np.zeros(128, dtype=np.float32)
    lib().hqref_dequantize_tile_rot(_ptr(a), lat, alpha, rp, seed, dither, e0, _ptr(out))
    return out


def rot_gaussian(seed: int, e: int) -> float:
    return float(lib().hqref_rot_gaussian(seed & (2**64 - 1), e & (2**64 - 1)))


# ---------------------------------------------------------------- whole tensors
def n_chunks(rows: int, cols: int) -> int:
    return int(lib().hqref_n_chunks(rows, cols))


def quantize(x, lat: int, alpha: float, k: int, seed: int, dither: int = 0, chunk_lo: int = 0,
             chunk_hi: int | None = None, dk_last: int = 0):
    """Weights path: bf16 [R, C] -> (stream words, offsets (n+1, relative), payload bits)."""
    xu = _as_u16(x)
    R, Cc = xu.shape
    if chunk_hi is None:
        chunk_hi = n_chunks(R, Cc)
    L = lib()
    off = np.zeros(chunk_hi - chunk_lo + 1, dtype=np.uint64)
    pb = np.zeros(1, dtype=np.uint64)
    total = int(L.hqref_quantize(_ptr(xu), R, Cc, Cc, lat, alpha, k, seed, dither, chunk_lo, chunk_hi, None, 0,
                                 _ptr(off), _ptr(pb), dk_last))
    total = abs(total)
    stream = np.zeros(max(total, 1), dtype=np.uint32)
    rc = int(L.hqref_quantize(_ptr(xu), R, Cc, Cc, lat, alpha, k, seed, dither, chunk_lo, chunk_hi,
                              _ptr(stream), stream.size, _ptr(off), _ptr(pb), dk_last))
    assert rc == total
    return stream[:total], off, int(pb[0])


def code_range(q):
    """[R11] (largest |q_i|, count of q_i outside [-128, 127]) over integer codes q."""
    a = np.ascontiguousarray(q, dtype=np.int32).ravel()
    mx = np.zeros(1, dtype=np.uint32)
    ov = np.zeros(1, dtype=np.uint64)
    lib().hqref_code_range(_ptr(a), a.size, _ptr(mx), _ptr(ov))
    return int(mx[0]), int(ov[0])


def quantize_range(x, lat: int, alpha: float, seed: int, dither: int = 0, chunk_lo: int = 0,
                   chunk_hi: int | None = None):
    """[R11] code range of the weights path's codes of chunks [chunk_lo, chunk_hi)."""
    xu = _as_u16(x)
    R, Cc = xu.shape
    if chunk_hi is None:
        chunk_hi = n_chunks(R, Cc)
    mx = np.zeros(1, dtype=np.uint32)
    ov = np.zeros(1, dtype=np.uint64)
    lib().hqref_quantize_range(_ptr(xu), R, Cc, Cc, lat, alpha, seed, dither, chunk_lo, chunk_hi, _ptr(mx), _ptr(ov))
    return int(mx[0]), int(ov[0])


def kv_range(kv, tok0: int, lat: int, alpha: float, seed: int, dither: int = 1, rot=None):
    """[R11] code range of one KV append's codes (bf16 [H, T, 128] at token tok0)."""
    r_keep, rp = _rot_ptr(rot)
    x = _as_u16(kv)
    H, T, D = x.shape
    assert D == 128
    mx = np.zeros(1, dtype=np.uint32)
    ov = np.zeros(1, dtype=np.uint64)
    lib().hqref_kv_range(_ptr(x), H, T, 128, T * 128, tok0, lat, alpha, seed, dither, rp, _ptr(mx), _ptr(ov))
    del r_keep
    return int(mx[0]), int(ov[0])


def dequantize(stream, offsets, rows: int, cols: int, lat: int, alpha: float, k: int, seed: int, dither: int = 0,
               out_fp32: bool = False, chunk_lo: int = 0, chunk_hi: int | None = None,
               out: np.ndarray | None = None, dk_last: int = 0) -> np.ndarray:
    """Weights path inverse: float32 [R, C] (fp32 mode) or uint16 bf16 bits [R, C].
    offsets[0] belongs to chunk chunk_lo; only that range's tiles of `out` are written."""
    if chunk_hi is None:
        chunk_hi = n_chunks(rows, cols)
    s = np.ascontiguousarray(stream, dtype=np.uint32)
    o = np.ascontiguousarray(offsets, dtype=np.uint64)
    if out is None:
        out = np.zeros((rows, cols), dtype=np.float32 if out_fp32 else np.uint16)
    assert out.shape == (rows, cols) and out.flags["C_CONTIGUOUS"]
    assert out.dtype == (np.float32 if out_fp32 else np.uint16)
    rc = lib().hqref_dequantize(_ptr(s), _ptr(o), rows, cols, lat, alpha, k, seed, dither, chunk_lo, chunk_hi,
                                int(out_fp32), _ptr(out), cols, dk_last)
    if rc != 0:
        raise ValueError("corrupt stream")
    return out


def _rot_ptr(rot):
    """A dense rotation as a C pointer (None: the sign diagonal and H_128)."""
    if rot is None:
        return None, None
    r = np.ascontiguousarray(rot, dtype=np.float32)
    assert r.shape == (128, 128)
    return r, _ptr(r)


def kv_append(kv, tok0: int, lat: int, alpha: float, k: int, seed: int, dither: int = 1, base_word: int = 0,
              rot=None, dk_last: int = 0):
    """One KV append: bf16 [H, T, 128] -> (stream words, absolute offsets (n+1), payload bits).
    rot: a 128 x 128 orthogonal fp32 matrix in place of H_128 D / sqrt(128), or None."""
    r_keep, rp = _rot_ptr(rot)
    x = _as_u16(kv)
    H, T, D = x.shape
    assert D == 128
    L = lib()
    nch = H * ((T + 31) // 32)
    off = np.zeros(nch + 1, dtype=np.uint64)
    pb = np.zeros(1, dtype=np.uint64)
    end = abs(int(L.hqref_kv_append(_ptr(x), H, T, 128, T * 128, tok0, lat, alpha, k, seed, dither, None,
                                    base_word, 0, _ptr(off), _ptr(pb), rp, dk_last)))
    total = end - base_word
    stream = np.zeros(max(end, 1), dtype=np.uint32)
    L.hqref_kv_append(_ptr(x), H, T, 128, T * 128, tok0, lat, alpha, k, seed, dither, _ptr(stream), base_word,
                      stream.size, _ptr(off), _ptr(pb), rp, dk_last)
    del r_keep
    return stream[base_word:end].copy(), off, int(pb[0])


def kv_read_append(stream_abs, offsets_abs, H: int, T: int, tok0: int, lat: int, alpha: float, k: int, seed: int,
                   dither: int, out: np.ndarray, length: int, rot=None, dk_last: int = 0):
    """Decode one append into out [H, len, 128] (float32 or uint16 bf16 bits)."""
    r_keep, rp = _rot_ptr(rot)
    s = np.ascontiguousarray(stream_abs, dtype=np.uint32)
    o = np.ascontiguousarray(offsets_abs, dtype=np.uint64)
    assert out.flags["C_CONTIGUOUS"] and out.shape[2] == 128
    rc = lib().hqref_kv_read_append(_ptr(s), _ptr(o), H, T, tok0, lat, alpha, k, seed, dither,
                                    int(out.dtype == np.float32), _ptr(out), 128, out.shape[1] * 128, length, rp,
                                    dk_last)
    del r_keep
    if rc != 0:
        raise ValueError("corrupt stream")
