"""hq_offsets_add on the GPU, and the partitioned path on one GPU: a set of matrices
coded in two blocks (as two ranks would), each block's offsets moved to its global
base, gives the offsets and words of the whole set coded in order by the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from hqtest import gpu_quantize

pytestmark = pytest.mark.gpu


def test_offsets_add():
    import lattice_entropy_coded_b200 as hq
    for n in (1, 7, 256, 100_003):
        off = torch.arange(n, dtype=torch.int64, device="cuda") * 3
        hq.hq_offsets_add(off, 1 << 40)
        torch.cuda.synchronize()
        assert torch.equal(off.cpu(), torch.arange(n, dtype=torch.int64) * 3 + (1 << 40))
    empty = torch.empty(0, dtype=torch.int64, device="cuda")
    hq.hq_offsets_add(empty, 5)


def test_two_blocks_assemble_into_one_stream():
    import lattice_entropy_coded_b200 as hq
    from lattice_entropy_coded_b200 import shard
    n, rows, cols, seed = 5, 96, 1024, 4
    mats = list(synth.student_t(n, rows, cols, seed))
    p = hq.make_params("E8", 355.45, 2, seed, 0)
    ref_w, ref_o, base = [], [], 0
    for m in mats:
        s, off, _ = O.quantize(m, O.E8, 355.45, 2, seed)
        ref_w.append(s[:int(off[-1])])
        ref_o.append(off[:-1].astype(np.uint64) + np.uint64(base))
        base += int(off[-1])
    ref_o.append(np.array([base], np.uint64))
    ref_w, ref_o = np.concatenate(ref_w), np.concatenate(ref_o)
    words, offs, gbase = [], [], 0
    for rank in range(2):
        lo, hi = shard.shard_range(n, 2, rank)
        local = 0
        for m in mats[lo:hi]:
            g = gpu_quantize(m.cuda(), p)
            o = g["offsets_t"].clone()
            hq.hq_offsets_add(o, gbase + local)
            torch.cuda.synchronize()
            words.append(g["words"])
            offs.append(o.cpu().numpy().view(np.uint64)[:-1])
            local += g["total"]
        gbase += local
    offs.append(np.array([gbase], np.uint64))
    assert np.array_equal(np.concatenate(words), ref_w)
    assert np.array_equal(np.concatenate(offs), ref_o)
