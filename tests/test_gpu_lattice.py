"""The device nearest-point decoders (the ones the quantize kernels inline) against
the oracle's, code for code, on the inputs where a decoder is easiest to get
wrong: points bisected onto the boundary between two Voronoi cells (with one
coordinate moved by one ulp either way), exact ties built from half-integers,
and magnitudes up to 2^21.  The E8 decoder decides between its two D8
candidates from a distance estimate with an error margin and falls back to the
sequential-fma distances inside it; boundary points are where that fallback
must take over, so they pin it.
"""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

LATS = {"Z": O.Z, "A2": O.A2, "D4": O.D4, "E8": O.E8}


def _device_codes(lat_name, v):
    import lattice_entropy_coded_b200 as hq
    vt = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).cuda()
    qt = torch.empty(vt.shape, dtype=torch.int32, device="cuda")
    hq.hq_debug_nearest(lat_name, vt, qt)
    torch.cuda.synchronize()
    return qt.cpu().numpy()


def _boundary_points(lat, dim, n, scale, rng, steps=48):
    """Points of a random segment a -> b (float32) next to where the oracle's code changes."""
    a = rng.uniform(-scale, scale, (n, dim)).astype(np.float32)
    b = (a + rng.uniform(-4.0, 4.0, (n, dim))).astype(np.float32)
    qa, qb = O.decode_many(lat, a), O.decode_many(lat, b)
    keep = np.any(qa != qb, axis=1)
    a, b, qa = a[keep], b[keep], qa[keep]
    lo, hi = np.zeros(len(a)), np.ones(len(a))
    for _ in range(steps):
        mid = (lo + hi) / 2
        m = (a + mid[:, None] * (b.astype(np.float64) - a)).astype(np.float32)
        same = np.all(O.decode_many(lat, m) == qa, axis=1)
        lo = np.where(same, mid, lo)
        hi = np.where(same, hi, mid)
    pts = []
    for t in (lo, hi):
        p = (a + t[:, None] * (b.astype(np.float64) - a)).astype(np.float32)
        pts.append(p)
        for direction in (np.inf, -np.inf):
            j = rng.integers(0, dim, len(p))
            q = p.copy()
            q[np.arange(len(p)), j] = np.nextafter(q[np.arange(len(p)), j], np.float32(direction))
            pts.append(q)
    return np.concatenate(pts)


def _tie_points(dim, n, rng):
    """Half-integer and quarter-integer vectors: many exact distance ties."""
    h = rng.integers(-8, 9, (n, dim)).astype(np.float32) * 0.5
    qtr = rng.integers(-16, 17, (n, dim)).astype(np.float32) * 0.25
    return np.concatenate([h, qtr, np.full((1, dim), 0.5, np.float32), np.zeros((1, dim), np.float32)])


@pytest.mark.parametrize("name", list(LATS))
def test_device_nearest_matches_oracle_on_boundaries_and_ties(name):
    lat = LATS[name]
    dim = O.DIM[lat]
    rng = np.random.default_rng(1000 + lat)
    parts = [_tie_points(dim, 20000, rng)]
    for scale in (0.5, 3.0, 20.0, 300.0, 2.0 ** 14, 2.0 ** 20):
        parts.append(_boundary_points(lat, dim, 6000, scale, rng))
        parts.append(rng.uniform(-scale, scale, (20000, dim)).astype(np.float32))
    v = np.concatenate(parts)
    want = O.decode_many(lat, v)
    got = _device_codes(name, v)
    bad = np.nonzero(np.any(got != want, axis=1))[0]
    assert len(bad) == 0, f"{len(bad)} of {len(v)} differ; first {v[bad[0]].tolist()}: {got[bad[0]]} vs {want[bad[0]]}"
