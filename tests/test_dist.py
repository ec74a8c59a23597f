"""The N > 1 path on CPU, with gloo ranks: the max over ranks of the step time, the
whole-job value, and the partition of a tensor set across ranks with the optional
global stream index (one all_gather of word counts, then a local offset add).

The coding itself has no exchange step: each rank codes its contiguous block of
the set on its own.  Here the ranks code their blocks with the oracle (the CPU
stands in for the GPUs), and the assembled global offsets must equal those of one
process coding the whole set in order."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)


def _timing_worker(rank, world, port, out):
    import bench
    _init(rank, world, port)
    try:
        times = [10.0 + 5.0 * rank, 3.0 - rank]          # rank 1 is slower in the first, faster in the second
        mx = bench.reduce_max(times, "cpu")
        sm = bench.reduce_sum([1e9 * (rank + 1)], "cpu")
        out[rank] = (mx, sm, bench.job_gbs(sm[0], mx[0]))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value():
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_timing_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        mx, sm, val = out[r]
        assert mx == [15.0, 3.0]
        assert sm == [3e9]
        assert val == pytest.approx(3e9 / (15.0 * 1e6))


def test_single_process_reduce_is_identity():
    import bench
    assert bench.reduce_max([1.5, 2.5], "cpu") == [1.5, 2.5]
    assert bench.reduce_sum([1.5, 2.5], "cpu") == [1.5, 2.5]
    assert bench.weak_scaling_value(1e9, 1, 1.0) == pytest.approx(1000.0)


@pytest.mark.parametrize("n,world", [(64, 1), (64, 2), (64, 8), (56, 3), (5, 2), (3, 4), (0, 2)])
def test_shard_range_covers_every_item_once_in_order(n, world):
    from lattice_entropy_coded_b200 import shard
    parts = [shard.shard_range(n, world, r) for r in range(world)]
    assert parts[0][0] == 0 and parts[-1][1] == n
    for (a, b), (c, d) in zip(parts, parts[1:]):
        assert b == c                                  # contiguous, in rank order
    sizes = [b - a for a, b in parts]
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == n
    with pytest.raises(ValueError):
        shard.shard_range(n, world, world)


SET = dict(n=5, rows=48, cols=384, seed=9, lat=3, alpha=300.0, k=2)    # E8


def _code_block(lo, hi):
    """The oracle's streams of matrices [lo, hi) of the set, concatenated: (words, offsets
    relative to the block's first word)."""
    import oracle as O
    import synth
    words, offs, base = [], [], 0
    for m in synth.student_t(hi - lo, SET["rows"], SET["cols"], SET["seed"], first=lo):
        s, off, _ = O.quantize(m, SET["lat"], SET["alpha"], SET["k"], SET["seed"])
        words.append(s[:int(off[-1])])
        offs.append(off[:-1].astype(np.uint64) + np.uint64(base))
        base += int(off[-1])
    offs.append(np.array([base], np.uint64))
    return (np.concatenate(words) if words else np.zeros(0, np.uint32)), np.concatenate(offs)


def _partition_worker(rank, world, port, out):
    from lattice_entropy_coded_b200 import shard
    _init(rank, world, port)
    try:
        lo, hi = shard.shard_range(SET["n"], world, rank)
        words, offs = _code_block(lo, hi)
        base, total = shard.global_base(int(offs[-1]), device="cpu")
        # what hq_offsets_add does on the device: every offset of this rank's part moves by base
        out[rank] = (lo, hi, words, offs + np.uint64(base), base, total)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_partitioned_set_assembles_into_one_global_stream(world):
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_partition_worker, args=(world, port, out), nprocs=world, join=True)
    ref_words, ref_offs = _code_block(0, SET["n"])
    parts = [out[r] for r in range(world)]
    assert [p[0] for p in parts] == sorted(p[0] for p in parts)
    words = np.concatenate([p[2] for p in parts])
    # each part's offsets without its end entry, then the last part's end: one offsets array
    offs = np.concatenate([p[3][:-1] for p in parts] + [parts[-1][3][-1:]])
    assert np.array_equal(words, ref_words)
    assert np.array_equal(offs, ref_offs)
    assert all(p[5] == len(ref_words) for p in parts)
    assert parts[0][4] == 0
