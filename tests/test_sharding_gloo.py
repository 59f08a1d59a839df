"""Multi-process (gloo, CPU) tests of the data-parallel sharding: two ranks split a batch by
batch element, each computes its part with the fp64 oracle, and the parts reassemble to the
single-process result; timing uses the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from hierarchical_chunk_sparse_scoring_b200 import sharding


def test_shard_range_covers_once():
    for n in range(0, 23):
        for world in range(1, 6):
            seen = []
            for r in range(world):
                a, b = sharding.shard_range(n, world, r)
                assert 0 <= a <= b <= n
                seen.extend(range(a, b))
            assert seen == list(range(n))
    with pytest.raises(ValueError):
        sharding.shard_range(4, 2, 2)


def test_aggregate_throughput():
    assert sharding.aggregate_tokens_per_s(1000, 2.0, 4) == pytest.approx(2e6)
    assert sharding.max_over_ranks(3.5) == 3.5          # no process group


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(0)          # same inputs on every rank
        B, Hq, Hkv, N, d, S = 5, 4, 2, 96, 8, 8
        C = N // S
        full = [torch.from_numpy(x) for x in (
            rng.standard_normal((B, Hq, N, d)), rng.standard_normal((B, Hq, N, d)),
            rng.standard_normal((B, Hkv, N, d)), rng.standard_normal((B, Hkv, N, d)),
            rng.standard_normal((B, Hkv, C, d)), rng.uniform(-1, 1, (B, Hkv, C)))]
        part = sharding.shard_batch(full, world, rank)
        r = oracle.forward(*[t.numpy() for t in part], S=S, K_top=3, W=12, threads=1)
        np.save(os.path.join(out_dir, "out_%d.npy" % rank), r["out"])
        np.save(os.path.join(out_dir, "idx_%d.npy" % rank), r["idx"])
        t = sharding.max_over_ranks(1.0 + rank)
        np.save(os.path.join(out_dir, "tmax_%d.npy" % rank), np.array([t]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_reassemble(tmp_path):
    import oracle
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    rng = np.random.default_rng(0)
    B, Hq, Hkv, N, d, S = 5, 4, 2, 96, 8, 8
    C = N // S
    arrs = (rng.standard_normal((B, Hq, N, d)), rng.standard_normal((B, Hq, N, d)),
            rng.standard_normal((B, Hkv, N, d)), rng.standard_normal((B, Hkv, N, d)),
            rng.standard_normal((B, Hkv, C, d)), rng.uniform(-1, 1, (B, Hkv, C)))
    ref = oracle.forward(*arrs, S=S, K_top=3, W=12, threads=1)
    out = np.concatenate([np.load(tmp_path / ("out_%d.npy" % r)) for r in range(world)])
    idx = np.concatenate([np.load(tmp_path / ("idx_%d.npy" % r)) for r in range(world)])
    np.testing.assert_array_equal(idx, ref["idx"])
    np.testing.assert_array_equal(out, ref["out"])
    for r in range(world):
        assert float(np.load(tmp_path / ("tmax_%d.npy" % r))[0]) == 2.0
