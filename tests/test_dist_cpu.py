"""Multi-rank host logic on the CPU (gloo, world size 2): token shards cover
the batch exactly, per-rank layers on their token shards reassemble the
single-rank result bit for bit (the path needs no exchange), and the
timing reduction takes the max over ranks."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from w4a4_int4_quantized_b200.shard import token_shard


@pytest.mark.parametrize("m,world", [(4608, 2), (4609, 2), (7, 4), (1, 3), (0, 2), (9216, 8)])
def test_token_shards_cover_the_batch(m, world):
    spans = [token_shard(m, world, r) for r in range(world)]
    pos = 0
    for start, count in spans:
        assert start == pos and count >= 0
        pos += count
    assert pos == m
    counts = [c for _, c in spans]
    assert max(counts) - min(counts) <= 1


def test_token_shard_rejects_bad_requests():
    with pytest.raises(ValueError):
        token_shard(10, 0, 0)
    with pytest.raises(ValueError):
        token_shard(10, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist

    import oracle
    from w4a4_int4_quantized_b200 import inputs
    from w4a4_int4_quantized_b200.shard import max_over_ranks, token_shard

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = inputs.LayerSpec("dist", 96, 256, 64, 64, rank=16, bias=True, seed=31, outlier_scale=100.0)
        d = inputs.make_layer(spec)           # every rank draws the same layer
        start, count = token_shard(spec.M, world, rank)
        ref = oracle.linear_w4a4(d["X"][start:start + count], d["W"], spec.group, d["L1"], d["L2"], d["bias"])
        y = torch.from_numpy(np.ascontiguousarray(ref["Y"]))
        codes = torch.from_numpy(ref["x_packed"].astype(np.int64))
        sizes = [None] * world
        dist.all_gather_object(sizes, count)
        ys = [torch.zeros((c, spec.N), dtype=torch.float64) for c in sizes]
        cs = [torch.zeros((c, spec.K // 2), dtype=torch.int64) for c in sizes]
        dist.all_gather(ys, y)
        dist.all_gather(cs, codes)
        t = max_over_ranks(1.0 + rank)
        if rank == 0:
            out.put((torch.cat(ys).numpy(), torch.cat(cs).numpy(), t))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_token_sharded_layer_matches_single_rank():
    import oracle
    from w4a4_int4_quantized_b200 import inputs

    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    y, codes, tmax = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    spec = inputs.LayerSpec("dist", 96, 256, 64, 64, rank=16, bias=True, seed=31, outlier_scale=100.0)
    d = inputs.make_layer(spec)
    full = oracle.linear_w4a4(d["X"], d["W"], spec.group, d["L1"], d["L2"], d["bias"])
    assert np.array_equal(codes, full["x_packed"].astype(np.int64))
    assert np.array_equal(y, full["Y"])
    assert tmax == 2.0
