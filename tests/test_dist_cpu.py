"""The multi-rank path on CPU (gloo, world size 2): batch-row sharding of the
layer, assembly by all-gather, and the max-over-ranks timing reduction.  The
per-rank compute here is the float64 oracle (no GPU on this machine); the
check is that the sharded result equals the unsharded one exactly."""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from compressive_memory_transformer_segment_b200 import shard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(5)  # same full problem on every rank
        B, H_q, H_kv, L, d = 3, 4, 2, 48, 8
        q = rng.standard_normal((B, H_q, L, d))
        k = rng.standard_normal((B, H_kv, L, d))
        v = rng.standard_normal((B, H_kv, L, d))
        beta = rng.uniform(-2, 2, H_q)
        M0 = np.zeros((B, H_kv, d, d))
        z0 = np.zeros((B, H_kv, d))
        b0, b1 = shard.batch_range(B, world, rank)
        out, M, z = oracle.infini_attention_forward(q[b0:b1], k[b0:b1], v[b0:b1], beta,
                                                    M0[b0:b1], z0[b0:b1], 16, "delta")
        full = [shard.gather_batch(torch.from_numpy(x), B, world) for x in (out, M, z)]
        ref = oracle.infini_attention_forward(q, k, v, beta, M0, z0, 16, "delta")
        ok = all(torch.equal(a, torch.from_numpy(r)) for a, r in zip(full, ref))
        mx = shard.max_over_ranks(10.0 + rank)
        results[rank] = (ok, mx, (b0, b1))
    finally:
        dist.destroy_process_group()


def test_batch_range_partition():
    for B in (1, 2, 3, 8, 17):
        for world in (1, 2, 3, 4, 8):
            rs = [shard.batch_range(B, world, r) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == B
            assert all(rs[i][1] == rs[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= 1


def test_two_rank_gloo_sharding_matches_single_process():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    mp.start_processes(_worker, args=(world, port, results), nprocs=world, join=True,
                       start_method="spawn")
    assert sorted(results.keys()) == [0, 1]
    for r in range(world):
        ok, mx, _ = results[r]
        assert ok
        assert mx == 11.0
    assert results[0][2] == (0, 2) and results[1][2] == (2, 3)
