"""Seeded synthetic inputs shaped like the HyperQuant pages' workloads.

This module holds input recipes only -- no step of the quantizer.  Both the
CUDA path (through the tests and the benchmark) and the CPU oracle receive
the tensors made here.

The pages evaluate on Llama-3.1-8B-Instruct weights and KV caches (WikiText-2)
and on the LTX-2 video DiT ("Experimental results" section); neither the
models nor the datasets are available, so these tensors stand in for them with
the shapes of an 8B model's linear layers and KV cache:

* ``weight``     -- bf16 N(0, 0.02^2) matrix with 0.1 % of positions, drawn
                    uniformly without replacement, scaled x20 (heavy outliers).
* ``kv``         -- K and V bf16 [heads, tokens, 128] N(0, 1); per head 4 K
                    channels drawn once and scaled x50 (outlier channels).
* ``weight_set`` -- 8 layers x {q 4096x4096, k 1024x4096, v 1024x4096,
                    o 4096x4096, gate/up 14336x4096, down 4096x14336 stored
                    transposed as 14336x4096}, N(0, 0.02^2).
* ``student_t``  -- matrices drawn from Student-t (nu = 5) scaled to std 0.02.

Every tensor is a pure function of (recipe, seed, device): CPU tensors come
from torch's CPU generator, CUDA tensors from torch's CUDA generator (the two
differ; a test that compares devices generates on the CPU and copies).
"""
from __future__ import annotations

import math

import torch

WEIGHT_STD = 0.02
OUTLIER_FRAC = 0.001
OUTLIER_SCALE = 20.0
KV_OUTLIER_CHANNELS = 4
KV_OUTLIER_SCALE = 50.0

# Shapes of one transformer layer of an 8B-class model (GQA with 8 KV heads).
LAYER_SHAPES = (
    ("q", 4096, 4096),
    ("k", 1024, 4096),
    ("v", 1024, 4096),
    ("o", 4096, 4096),
    ("gate", 14336, 4096),
    ("up", 14336, 4096),
    ("down_t", 14336, 4096),
)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weight(rows: int, cols: int, seed: int, device="cpu", std: float = WEIGHT_STD,
           outlier_frac: float = OUTLIER_FRAC, outlier_scale: float = OUTLIER_SCALE) -> torch.Tensor:
    """bf16 [rows, cols] ~ N(0, std^2) with round(frac*n) uniformly placed positions scaled."""
    g = _gen(seed, device)
    w = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32).mul_(std)
    n = rows * cols
    n_out = int(round(outlier_frac * n))
    if n_out:
        idx = torch.randperm(n, generator=g, device=device)[:n_out]
        w.view(-1)[idx] *= outlier_scale
    return w.to(torch.bfloat16)


def kv(heads: int, tokens: int, seed: int, device="cpu", head_dim: int = 128):
    """(K, V) bf16 [heads, tokens, head_dim] ~ N(0, 1); 4 K channels per head scaled x50."""
    g = _gen(seed, device)
    k = torch.randn(heads, tokens, head_dim, generator=g, device=device, dtype=torch.float32)
    v = torch.randn(heads, tokens, head_dim, generator=g, device=device, dtype=torch.float32)
    for h in range(heads):
        ch = torch.randperm(head_dim, generator=g, device=device)[:KV_OUTLIER_CHANNELS]
        k[h, :, ch] *= KV_OUTLIER_SCALE
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


def weight_set(seed: int, device="cpu", layers: int = 8, std: float = WEIGHT_STD):
    """Yields (name, bf16 matrix) for every linear weight of `layers` layers, no outliers."""
    g = _gen(seed, device)
    for layer in range(layers):
        for name, r, c in LAYER_SHAPES:
            w = torch.randn(r, c, generator=g, device=device, dtype=torch.float32).mul_(std)
            yield f"layer{layer}.{name}", w.to(torch.bfloat16)


def weight_set_elems(layers: int = 8) -> int:
    return layers * sum(r * c for _, r, c in LAYER_SHAPES)


STUDENT_T_STRIDE = 1_000_003   # matrix i of a set is drawn from seed + i * STUDENT_T_STRIDE


def student_t(n: int, rows: int, cols: int, seed: int, device="cpu", nu: int = 5, std: float = WEIGHT_STD,
              first: int = 0):
    """Yields n bf16 matrices (numbers first .. first + n - 1 of the set), entries
    Student-t(nu) * std / sqrt(nu / (nu - 2)) (so std = `std`).  Each matrix has its
    own generator, so any part of the set can be drawn alone (one rank's share).

    t = N / sqrt(chi2_nu / nu) with chi2_nu a sum of nu squared standard normals."""
    scale = std / math.sqrt(nu / (nu - 2.0))
    for i in range(first, first + n):
        g = _gen(seed + i * STUDENT_T_STRIDE, device)
        z = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
        chi2 = torch.zeros_like(z)
        for _ in range(nu):
            e = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
            chi2.addcmul_(e, e)
        t = z.div_(chi2.div_(nu).sqrt_()).mul_(scale)
        yield t.to(torch.bfloat16)


# The five workloads, named by what they are.
WORKLOADS = {
    "weight_1024x1024_e8_4bps": dict(kind="weight", rows=1024, cols=1024, seed=0),
    "weight_4096x4096_rate_sweep": dict(kind="weight", rows=4096, cols=4096, seed=1),
    # the same sweep with a second Rice parameter for the last symbol of each block
    "weight_4096x4096_rate_sweep_dk": dict(kind="weight", rows=4096, cols=4096, seed=1,
                                           points_of="weight_4096x4096_rate_sweep",
                                           dk_last={"E8": 1, "D4": 1, "A2": 2, "Z": 0}),
    "kv_8h_32768tok_e8_dither": dict(kind="kv", heads=8, tokens=32768, seed=2, append=256),
    # the same cache with a dense Haar-uniform rotation per tensor instead of the sign diagonal and H_128
    "kv_8h_32768tok_e8_dither_haar": dict(kind="kv", heads=8, tokens=32768, seed=2, append=256, rotation=True),
    "weights_8b_8layers_e8_4bps": dict(kind="weight_set", layers=8, seed=3),
    "student_t_64x8192x8192_e8": dict(kind="student_t", n=64, rows=8192, cols=8192, seed=4),
}
