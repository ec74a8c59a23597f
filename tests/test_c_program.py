"""libhq.so from C programs that include include/hq.h and the CUDA runtime only:
tests/c/hq_roundtrip.c (a weight matrix: quantize, rate, dequantize, fused GEMV) and
tests/c/hq_kv_roundtrip.c (a KV cache with a dense rotation, dither and a second Rice
parameter, and the library's Haar draw).  They compile and link here (no GPU needed);
on a GPU their outputs are compared with the oracle."""
import json
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle as O
import synth
from hqtest import assert_recon_equal, oracle_dequantize, oracle_quantize, u16
from oracle import rotation as R

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "lattice_entropy_coded_b200")
CUDA = "/usr/local/cuda"


def _compile(out_dir, name="hq_roundtrip") -> str:
    exe = os.path.join(str(out_dir), name)
    cmd = ["gcc", "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c", name + ".c"),
           "-L", PKG, "-lhq", "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{PKG}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


@pytest.mark.parametrize("name", ["hq_roundtrip", "hq_kv_roundtrip"])
def test_c_program_compiles_and_links(tmp_path, name):
    exe = _compile(tmp_path, name)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 1 and "usage" in r.stderr      # runs (library resolved), prints usage


@pytest.mark.gpu
def test_c_program_matches_the_oracle(tmp_path):
    exe = _compile(tmp_path)
    rows, cols, seed, alpha, k = 37, 384, 5, 314.1544494628906, 2
    W = synth.weight(rows, cols, seed=41)
    v = (torch.randn(cols, generator=torch.Generator().manual_seed(3)) * 0.7).to(torch.bfloat16)
    inp = tmp_path / "in.bin"
    inp.write_bytes(u16(W).tobytes() + u16(v).tobytes())
    prefix = str(tmp_path / "out_")
    r = subprocess.run([exe, str(inp), str(rows), str(cols), str(O.E8), repr(alpha), str(k), str(seed), prefix],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    info = json.loads(r.stdout)
    ref_w, ref_off, ref_pay = oracle_quantize(W, O.E8, alpha, k, seed)
    assert info["payload_bits"] == ref_pay and info["stream_words"] == len(ref_w)
    assert np.array_equal(np.fromfile(prefix + "stream.bin", np.uint32), ref_w)
    assert np.array_equal(np.fromfile(prefix + "offsets.bin", np.uint64), ref_off)
    ref_out = oracle_dequantize(ref_w, ref_off, rows, cols, O.E8, alpha, k, seed, fp32=False)
    assert np.array_equal(np.fromfile(prefix + "out.bin", np.uint16).reshape(rows, cols), ref_out)
    w = (ref_out.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    x = (u16(v).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    y = np.fromfile(prefix + "y.bin", np.float32).astype(np.float64)
    lim = (40 + cols // 128) * 2.0 ** -24 * (np.abs(w) @ np.abs(x)) + 1e-30
    assert np.all(np.abs(y - w @ x) <= lim)


@pytest.mark.gpu
def test_c_kv_program_matches_the_oracle(tmp_path):
    exe = _compile(tmp_path, "hq_kv_roundtrip")
    H, t1, t2, alpha, k, dk, seed = 3, 70, 45, 0.6, 1, 1, 29
    K, _ = synth.kv(H, t1 + t2, seed=42)
    Q = R.haar_rotation(seed)
    (tmp_path / "in.bin").write_bytes(u16(K).tobytes())
    (tmp_path / "q.bin").write_bytes(Q.tobytes())
    prefix = str(tmp_path / "kv_")
    r = subprocess.run([exe, str(tmp_path / "in.bin"), str(tmp_path / "q.bin"), str(H), str(t1), str(t2), repr(alpha),
                        str(k), str(dk), str(seed), prefix], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    info = json.loads(r.stdout)
    assert info["appends"] == 2
    words, offs, base, pay = [], [], 0, 0
    ref = np.zeros((H, t1 + t2, 128), np.float32)
    for t0, T in ((0, t1), (t1, t2)):
        a = K[:, t0:t0 + T].contiguous()
        s_, off, pb = O.kv_append(a, t0, O.E8, alpha, k, seed, 1, base_word=base, rot=Q, dk_last=dk)
        O.kv_read_append(s_, off - np.uint64(base), H, T, t0, O.E8, alpha, k, seed, 1, ref, t1 + t2, rot=Q, dk_last=dk)
        words.append(s_)
        offs.append(off[:-1])
        base = int(off[-1])
        pay += pb
    offs.append(np.array([base], np.uint64))
    assert info["payload_bits"] == pay and info["stream_words"] == base
    assert np.array_equal(np.fromfile(prefix + "stream.bin", np.uint32), np.concatenate(words))
    assert np.array_equal(np.fromfile(prefix + "offsets.bin", np.uint64), np.concatenate(offs))
    assert_recon_equal(np.fromfile(prefix + "out.bin", np.float32).reshape(H, t1 + t2, 128), ref)
    d = (np.fromfile(prefix + "qdraw.bin", np.float32).reshape(128, 128).view(np.int32).astype(np.int64)
         - Q.view(np.int32).astype(np.int64))
    assert np.abs(d).max() <= 1          # the library's Haar draw: the oracle's to one ulp
