"""World-size-2 checks of the data-parallel host logic on CPU (gloo).

Each rank quantizes its own token shard with the CPU oracle; gathering the
shards reproduces the single-process result bit for bit (units are
independent, so the path needs no data exchange), and the timing reduction
takes the slowest rank.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from block_floating_point_hif4_b200 import sharding


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist

    import oracle
    from block_floating_point_hif4_b200 import workloads as wl
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = wl.quant_sweep(1 << 16).reshape(-1, 1024)
        a, b = sharding.token_shard(x.shape[0], world, rank)
        codes, meta, _ = oracle.quantize(x[a:b])
        parts_c = [None] * world
        parts_m = [None] * world
        dist.all_gather_object(parts_c, codes)
        dist.all_gather_object(parts_m, meta)
        slowest = sharding.max_over_ranks(1.0 + rank)
        sharding.barrier()
        if rank == 0:
            out.put((np.concatenate(parts_c), np.concatenate(parts_m), slowest))
    finally:
        dist.destroy_process_group()


def test_token_shard_partition():
    for total in [0, 1, 7, 57600, 57601]:
        for world in [1, 2, 3, 8]:
            spans = [sharding.token_shard(total, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        sharding.token_shard(10, 2, 2)


def test_aggregate_throughput():
    assert sharding.aggregate_throughput(10.0, 4, 2.0) == 20.0
    assert sharding.rank_seed(3, 0) == 3 and sharding.rank_seed(3, 1) != sharding.rank_seed(3, 0)


def test_two_ranks_gloo_sharded_quantize_equals_whole():
    import oracle
    from block_floating_point_hif4_b200 import workloads as wl
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    codes, meta, slowest = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = wl.quant_sweep(1 << 16).reshape(-1, 1024)
    rc, rm, _ = oracle.quantize(x)
    assert np.array_equal(codes, rc) and np.array_equal(meta, rm)
    assert slowest == 2.0
