"""libhq.so from a C program: tests/c/hq_roundtrip.c includes include/hq.h and the
CUDA runtime only.  It compiles and links here (no GPU needed); on a GPU its
stream, offsets, bf16 reconstruction and fused GEMV are compared with the oracle."""
import json
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle as O
import synth
from hqtest import oracle_dequantize, oracle_quantize, u16

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "lattice_entropy_coded_b200")
CUDA = "/usr/local/cuda"


def _compile(out_dir) -> str:
    exe = os.path.join(str(out_dir), "hq_roundtrip")
    cmd = ["gcc", "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c", "hq_roundtrip.c"),
           "-L", PKG, "-lhq", "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{PKG}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_c_program_compiles_and_links(tmp_path):
    exe = _compile(tmp_path)
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
