"""The C-ABI library loads on a machine without a GPU, exports every entry point
include/hq.h declares, and its host-side logic (sizes, argument checks) is
right.  No compute call is made here."""
import ctypes as C
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "hq.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"HQ_API\s+(?:const\s+)?\w+\s*\*?\s*(hq_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("hq_quantize", "hq_dequantize", "hq_kv_append", "hq_kv_read", "hq_stream_bound",
              "hq_workspace_bytes", "hq_kv_init", "hq_status_string", "hq_device_check"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import lattice_entropy_coded_b200 as hq
    lib = C.CDLL(hq.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
        assert name in hq.EXPORTS, f"binding misses {name}"


def test_struct_layouts_match_header():
    import lattice_entropy_coded_b200 as hq
    assert C.sizeof(hq.hq_params) == 48
    assert hq.hq_params.seed.offset == 16 and hq.hq_params.chunk_tiles.offset == 28
    assert hq.hq_params.rotation.offset == 32 and hq.hq_params.rice_dk_last.offset == 40
    assert C.sizeof(hq.hq_stats) == 40 and hq.hq_stats.payload_bits.offset == 8
    assert hq.hq_stats.max_abs_code.offset == 24 and hq.hq_stats.int8_overflow_count.offset == 32
    assert C.sizeof(hq.hq_kv_append_row) == 32
    assert C.sizeof(hq.hq_kv_cache) == 144 and hq.hq_kv_cache.params.offset == 72
    assert hq.hq_kv_cache.tokens.offset == 120
    assert C.sizeof(hq.hq_calib_spec) == 48 and hq.hq_calib_spec.k_lo.offset == 32
    assert C.sizeof(hq.hq_calib_result) == 24 and hq.hq_calib_result.bps.offset == 8


def test_stream_bound_and_workspace():
    import lattice_entropy_coded_b200 as hq
    p = hq.make_params("E8", 300.0, 2)
    w, n = hq.hq_stream_bound(1024, 1024, p, 255)
    assert n == 256
    # per chunk: 16 coset words + 4*2*32 remainder words + 4096 * (1 + 511 >> 2) bits
    assert w == 256 * (16 + 256 + 4096 * (1 + (511 >> 2)) // 32)
    w2, n2 = hq.hq_stream_bound(3, 384, p, 7)      # 9 tiles: one partial chunk
    assert n2 == 1
    assert w2 == math.ceil(16 * 9 / 32) + 4 * 2 * 9 + math.ceil(9 * 128 * (1 + (15 >> 2)) / 32)
    assert hq.hq_stream_bound(0, 4096, p) == (0, 0)
    # a second Rice parameter for the last symbol of each block: 1 in 8 E8 symbols at k - 1
    p2 = hq.make_params("E8", 300.0, 2, dk_last=1)
    w3, _ = hq.hq_stream_bound(3, 384, p2, 7)
    assert w3 == (math.ceil(16 * 9 / 32) + math.ceil((1008 * 2 + 144 * 1) / 32)
                  + math.ceil((1008 * (1 + (15 >> 2)) + 144 * (1 + (15 >> 1))) / 32))
    assert hq.hq_workspace_bytes(1000) >= 1000 * 8 + 8
    assert hq.hq_workspace_bytes(1000) % 256 == 0


@pytest.mark.parametrize("bad", [
    dict(lattice=7), dict(alpha=0.0), dict(alpha=float("nan")), dict(alpha=-1.0), dict(rice_k=16),
    dict(rice_k=-1), dict(dither=2), dict(dk_last=-1), dict(dk_last=16)])
def test_invalid_params_rejected(bad):
    import lattice_entropy_coded_b200 as hq
    kw = dict(lattice=3, alpha=1.0, rice_k=2, seed=0, dither=0, dk_last=0)
    kw.update(bad)
    p = hq.hq_params(128, kw["lattice"], kw["alpha"], kw["rice_k"], 0, kw["dither"], 32, None, kw["dk_last"], 0)
    with pytest.raises(hq.HQError, match="invalid"):
        hq.hq_stream_bound(32, 128, p)


def test_unsupported_shapes_rejected():
    import lattice_entropy_coded_b200 as hq
    p = hq.make_params()
    p.tile = 64
    with pytest.raises(hq.HQError, match="unsupported"):
        hq.hq_stream_bound(32, 128, p)
    p = hq.make_params()
    p.chunk_tiles = 16
    with pytest.raises(hq.HQError, match="unsupported"):
        hq.hq_stream_bound(32, 128, p)
    p = hq.make_params()
    with pytest.raises(hq.HQError, match="invalid"):
        hq.hq_stream_bound(32, 100, p)          # cols not a multiple of 128
    with pytest.raises(hq.HQError, match="unsupported"):
        hq.hq_stream_bound(1, 128 * 1024, p)    # sign table too wide


def _no_device_or_skip():
    """Some checks below pass made-up device addresses and rely on the argument checks
    returning before any launch.  Where a GPU is present, a regression in those checks
    would launch a kernel on them, so these cases run only where no CUDA device is
    visible (the tests' CPU tier)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("made-up device addresses: run only without a CUDA device")


def test_entry_points_validate_before_touching_the_device():
    """Null or misaligned pointers come back as HQ_EINVAL with no CUDA call made."""
    _no_device_or_skip()
    import lattice_entropy_coded_b200 as hq
    lib = hq._lib
    p = hq.make_params()
    off = C.c_uint64()
    # misaligned offsets
    assert lib.hq_quantize(None, 32, 128, 128, C.byref(p), None, 0, 3, None, None, 0, None) == hq.HQ_EINVAL
    assert lib.hq_dequantize(None, 0, None, 32, 128, C.byref(p), None, 0, 128, None, None) == hq.HQ_EINVAL
    assert lib.hq_dequantize(None, 0, None, 32, 128, C.byref(p), None, 2, 128, None, None) == hq.HQ_EINVAL
    cache = hq.hq_kv_cache()
    assert lib.hq_kv_init(C.byref(cache), 8, 64, C.byref(p), None, 0, None, 0, None, 0, None, None,
                          None) == hq.HQ_EUNSUPPORTED
    assert lib.hq_kv_append(C.byref(cache), None, 16, 128, 2048, C.c_float(1.0), None, 0, None) == hq.HQ_EINVAL
    assert lib.hq_kv_read(C.byref(cache), None, 0, 1, 128, 2048, None) == hq.HQ_EINVAL
    assert hq.hq_status_string(hq.HQ_ST_TIMEOUT) == "look-back timed out"
    # rate and calibration: argument errors before any device work
    st = C.c_void_p(64)
    assert lib.hq_rate(None, 32, 128, 128, C.byref(p), st, None) == hq.HQ_EINVAL          # null x
    assert lib.hq_rate(None, 32, 100, 128, C.byref(p), st, None) == hq.HQ_EINVAL          # cols % 128
    assert lib.hq_rate(None, 32, 128, 128, C.byref(p), None, None) == hq.HQ_EINVAL        # null stats
    assert lib.hq_rate_kv(None, 0, 16, 128, 2048, 0, C.byref(p), st, None) == hq.HQ_EINVAL  # heads 0
    assert lib.hq_rate_kv(None, 8, 16, 128, 2048, -1, C.byref(p), st, None) == hq.HQ_EINVAL  # tok0 < 0
    res = hq.hq_calib_result()
    good = hq.calib_spec(4.0)
    assert lib.hq_calibrate(None, 32, 128, 128, C.byref(p), C.byref(good), st, None, C.byref(res)) == hq.HQ_EINVAL
    for bad in (hq.calib_spec(0.0), hq.calib_spec(4.0, alpha_lo=2.0, alpha_hi=1.0), hq.calib_spec(4.0, k_lo=3, k_hi=2),
                hq.calib_spec(4.0, k_hi=16), hq.calib_spec(4.0, tol=-1.0), hq.calib_spec(4.0, max_iter=201)):
        assert lib.hq_calibrate(C.c_void_p(256), 32, 128, 128, C.byref(p), C.byref(bad), st, None,
                                C.byref(res)) == hq.HQ_EINVAL
    assert lib.hq_calibrate(C.c_void_p(256), 0, 128, 128, C.byref(p), C.byref(good), st, None,
                            C.byref(res)) == hq.HQ_EINVAL                                   # empty
    # testing aids: encoder form switch and the nearest-point entry point
    assert lib.hq_debug_set_encode_path(5) == hq.HQ_EINVAL
    assert lib.hq_debug_set_encode_path(4) == hq.HQ_OK
    assert lib.hq_debug_set_encode_path(-1) == hq.HQ_EINVAL
    assert lib.hq_debug_set_encode_path(0) == hq.HQ_OK
    assert lib.hq_debug_nearest(4, None, 1, None, None) == hq.HQ_EINVAL
    assert lib.hq_debug_nearest(3, None, -1, None, None) == hq.HQ_EINVAL
    assert lib.hq_debug_nearest(3, None, 0, None, None) == hq.HQ_OK
    assert lib.hq_debug_nearest(3, None, 5, None, None) == hq.HQ_EINVAL


def test_dense_rotation_is_a_kv_option():
    """The weights entry points refuse a dense rotation (HQ_EUNSUPPORTED) and every entry
    point refuses a misaligned one (HQ_EINVAL), before any device work."""
    _no_device_or_skip()
    import lattice_entropy_coded_b200 as hq
    lib = hq._lib
    p = hq.make_params()
    p.rotation = 4096
    st = C.c_void_p(64)
    res = hq.hq_calib_result()
    good = hq.calib_spec(4.0)
    assert lib.hq_quantize(C.c_void_p(256), 32, 128, 128, C.byref(p), C.c_void_p(256), 64, C.c_void_p(256), None,
                           C.c_void_p(256), 1 << 20, None) == hq.HQ_EUNSUPPORTED
    assert lib.hq_quantize_static(C.c_void_p(256), 32, 128, 128, C.byref(p), C.c_void_p(256), 64, C.c_void_p(256),
                                  None, None) == hq.HQ_EUNSUPPORTED
    assert lib.hq_dequantize(C.c_void_p(256), 64, C.c_void_p(256), 32, 128, C.byref(p), C.c_void_p(256), 0, 128,
                             None, None) == hq.HQ_EUNSUPPORTED
    assert lib.hq_rate(C.c_void_p(256), 32, 128, 128, C.byref(p), st, None) == hq.HQ_EUNSUPPORTED
    assert lib.hq_calibrate(C.c_void_p(256), 32, 128, 128, C.byref(p), C.byref(good), st, None,
                            C.byref(res)) == hq.HQ_EUNSUPPORTED
    assert lib.hq_gemv(C.c_void_p(256), 64, C.c_void_p(256), 32, 128, C.byref(p), C.c_void_p(256),
                       C.c_void_p(256), C.c_void_p(256), 1 << 20, None, None) == hq.HQ_EUNSUPPORTED
    p.rotation = 4100                    # not 16-byte aligned
    cache = hq.hq_kv_cache()
    assert lib.hq_kv_init(C.byref(cache), 8, 128, C.byref(p), C.c_void_p(256), 64, C.c_void_p(256), 8,
                          C.c_void_p(256), 8, C.c_void_p(256), C.c_void_p(256), None) == hq.HQ_EINVAL
    assert lib.hq_rate_kv(C.c_void_p(256), 8, 16, 128, 2048, 0, C.byref(p), st, None) == hq.HQ_EINVAL
    assert lib.hq_haar_rotation(1, None, None) == hq.HQ_EINVAL
    assert lib.hq_haar_rotation(1, C.c_void_p(4100), None) == hq.HQ_EINVAL


def test_static_entry_point_applies_the_same_checks():
    """hq_quantize_static rejects what hq_quantize rejects (the shared argument checks),
    including a row count whose rows * (cols / 128) would wrap, and sizes beyond its
    fixed scratch; null pointers only, so nothing can reach a device."""
    import lattice_entropy_coded_b200 as hq
    lib = hq._lib
    p = hq.make_params("E8", 300.0, 2)
    cases = [  # rows, cols, hq_quantize_static, hq_quantize (null pointers)
        (1 << 55, 65536, hq.HQ_EUNSUPPORTED, hq.HQ_EUNSUPPORTED),
        (32, 100, hq.HQ_EINVAL, hq.HQ_EINVAL),
        (32, 131072, hq.HQ_EUNSUPPORTED, hq.HQ_EUNSUPPORTED),
        (hq.HQ_STATIC_MAX_CHUNKS + 1, 4096, hq.HQ_EUNSUPPORTED, hq.HQ_EINVAL),
        (hq.HQ_STATIC_MAX_CHUNKS, 4096, hq.HQ_EINVAL, hq.HQ_EINVAL),
        (-1, 128, hq.HQ_EINVAL, hq.HQ_EINVAL),
    ]
    for rows, cols, want_static, want in cases:
        assert lib.hq_quantize_static(None, rows, cols, cols, C.byref(p), None, 0, None, None, None) == want_static
        assert lib.hq_quantize(None, rows, cols, cols, C.byref(p), None, 0, None, None, None, 0, None) == want
    bad = hq.make_params("E8", 300.0, 2)
    bad.rice_k = 16
    assert lib.hq_quantize_static(None, 32, 128, 128, C.byref(bad), None, 0, None, None, None) == hq.HQ_EINVAL
    p.rotation = 4096
    assert lib.hq_quantize_static(None, 32, 128, 128, C.byref(p), None, 0, None, None, None) == hq.HQ_EUNSUPPORTED


def test_batch_entry_points_check_their_arguments():
    """Strided batches: sizes and argument errors, all before any device work (null pointers only)."""
    import lattice_entropy_coded_b200 as hq
    lib = hq._lib
    p = hq.make_params("E8", 300.0, 2)
    assert hq.hq_batch_workspace_bytes(64, 16384) >= 64 * 16384 * 8 + 8 + 64 * hq.STATS_BYTES
    assert hq.hq_batch_workspace_bytes(64, 16384) % 256 == 0
    assert hq.hq_batch_workspace_bytes(0, 16384) >= 8
    q = lambda *a: lib.hq_quantize_batch(*a)
    # batch < 0; batch * chunks beyond 2^31; batch 0 is a no-op
    assert q(None, -1, 0, 32, 128, 128, C.byref(p), None, 0, 0, None, None, None, 0, None) == hq.HQ_EINVAL
    assert q(None, 1 << 30, 0, 4096, 4096, 4096, C.byref(p), None, 0, 0, None, None, None, 0,
             None) == hq.HQ_EUNSUPPORTED
    assert q(None, 0, 0, 32, 128, 128, C.byref(p), None, 0, 0, None, None, None, 0, None) == hq.HQ_OK
    # batch >= 2 with null buffers or strides that overlap the items
    assert q(None, 2, 4096, 32, 128, 128, C.byref(p), None, 100, 100, None, None, None, 0, None) == hq.HQ_EINVAL
    d = lambda *a: lib.hq_dequantize_batch(*a)
    assert d(None, 0, 0, None, -1, 32, 128, C.byref(p), None, 0, 128, 4096, None, None) == hq.HQ_EINVAL
    assert d(None, 0, 0, None, 0, 32, 128, C.byref(p), None, 0, 128, 4096, None, None) == hq.HQ_OK
    assert d(None, 10, 5, None, 3, 32, 128, C.byref(p), None, 0, 128, 4096, None, None) == hq.HQ_EINVAL
    assert d(None, 10, 5, None, 3, 32, 128, C.byref(p), None, 2, 128, 4096, None, None) == hq.HQ_EINVAL


def test_binding_fails_loudly_without_the_library(tmp_path):
    """The binding has no fallback: a missing libhq.so is an import error."""
    import subprocess
    import sys
    pkg = tmp_path / "lattice_entropy_coded_b200"
    pkg.mkdir()
    with open(os.path.join(ROOT, "lattice_entropy_coded_b200", "__init__.py")) as f:
        (pkg / "__init__.py").write_text(f.read())
    r = subprocess.run([sys.executable, "-c", "import lattice_entropy_coded_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libhq.so is missing" in r.stderr
