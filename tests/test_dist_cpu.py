"""The multi-rank path on CPU (gloo, world size 2): batch-row sharding of the
layer, assembly by all-gather, and the max-over-ranks timing reduction.  The
per-rank compute here is the float64 oracle (no GPU on this machine); the
check is that the sharded result equals the unsharded one exactly."""

import os
import socket

import numpy as np
import pytest
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


# ------------------------------------------- (batch row, KV head) chain blocks

def test_chain_blocks_tile_the_grid():
    for B, H_kv in ((1, 32), (2, 8), (1, 4), (2, 3), (8, 12), (4, 16), (3, 5)):
        for world in range(1, 17):
            try:
                blocks = [shard.chain_block(B, H_kv, world, r) for r in range(world)]
            except ValueError:
                assert world > B * H_kv or all(world % wh or world // wh > B
                                               for wh in range(1, min(world, H_kv) + 1))
                continue
            seen = np.zeros((B, H_kv), dtype=int)
            for b0, b1, h0, h1 in blocks:
                assert b1 > b0 and h1 > h0
                seen[b0:b1, h0:h1] += 1
            assert np.all(seen == 1), (B, H_kv, world)
    # One long stream (B = 1) splits over its KV heads; exact splits come first.
    assert shard.split_factors(1, 32, 8) == (1, 8)
    assert shard.split_factors(2, 8, 16) == (2, 8)
    assert shard.split_factors(2, 3, 2) == (2, 1)


_CHAIN_CASES = {"one_stream": (1, 8, 4), "two_rows": (2, 6, 3)}  # (B, H_q, H_kv)


def _chain_worker(rank, world, port, case, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H_q, H_kv = _CHAIN_CASES[case]
        L, d, S, g = 40, 8, 16, H_q // H_kv
        rng = np.random.default_rng(11)  # same full problem on every rank
        q = rng.standard_normal((B, H_q, L, d))
        k = rng.standard_normal((B, H_kv, L, d))
        v = rng.standard_normal((B, H_kv, L, d))
        beta = rng.uniform(-2, 2, H_q)
        M0 = rng.standard_normal((B, H_kv, d, d))
        z0 = rng.uniform(0.5, 2.0, (B, H_kv, d))
        block = shard.chain_block(B, H_kv, world, rank)
        t = torch.from_numpy
        h0, h1 = block[2], block[3]
        out, M, z = oracle.infini_attention_forward(
            shard.shard_chains(t(q), block, g).numpy(), shard.shard_chains(t(k), block).numpy(),
            shard.shard_chains(t(v), block).numpy(), beta[h0 * g:h1 * g],
            shard.shard_chains(t(M0), block).numpy(), shard.shard_chains(t(z0), block).numpy(),
            S, "delta")
        full = (shard.gather_chains(t(out), B, H_kv, world, g), shard.gather_chains(t(M), B, H_kv, world),
                shard.gather_chains(t(z), B, H_kv, world))
        ref = oracle.infini_attention_forward(q, k, v, beta, M0, z0, S, "delta")
        results[rank] = (all(torch.equal(a, t(r)) for a, r in zip(full, ref)), block)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case,world", [("one_stream", 2), ("one_stream", 3), ("two_rows", 2),
                                        ("two_rows", 3)])
def test_chain_block_sharding_gloo(case, world):
    """Every rank runs the layer (float64 oracle as the per-rank compute) on its
    block of (batch row, KV head) chains, with the query heads of its groups;
    the gathered output and final state equal the single-process forward
    exactly."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    mp.start_processes(_chain_worker, args=(world, port, case, results), nprocs=world, join=True,
                       start_method="spawn")
    assert sorted(results.keys()) == list(range(world))
    for r in range(world):
        ok, block = results[r]
        assert ok, (r, block)
    if case == "one_stream":  # B = 1: the split is over KV heads
        assert all(results[r][1][:2] == (0, 1) for r in range(world))


# ------------------------------------------- sequence parallelism (linear rule)

def _oracle_forward(q, k, v, beta, M_in, z_in, S, rule):
    out, M, z = oracle.infini_attention_forward(q.numpy(), k.numpy(), v.numpy(), beta.numpy(),
                                                M_in.numpy(), z_in.numpy(), S, rule)
    return torch.from_numpy(out), torch.from_numpy(M), torch.from_numpy(z)


def _oracle_state_update(k, v, M_in, z_in, S, rule):
    B, H_kv, L, d_k = k.shape
    q = torch.zeros((B, H_kv, L, d_k), dtype=torch.float64)
    beta = torch.zeros(H_kv, dtype=torch.float64)
    _, M, z = _oracle_forward(q, k, v, beta, M_in, z_in, S, rule)
    return M, z


def _host_state_sum(M_base, z_base, parts, n_parts):
    """The sum the library's state_sum forms, on host tensors (test stand-in
    for the CUDA call): base plus the first n_parts packed states, in order."""
    nM = M_base.numel()
    M, z = M_base.clone(), z_base.clone()
    for p in range(n_parts):
        M += parts[p, :nM].view_as(M)
        z += parts[p, nM:].view_as(z)
    return M, z


def _sp_problem():
    # 7 segments of 16 rows, the last one 4 rows; GQA; a nonzero initial state.
    rng = np.random.default_rng(9)
    B, H_q, H_kv, L, d, S = 2, 4, 2, 100, 8, 16
    q = rng.standard_normal((B, H_q, L, d))
    k = rng.standard_normal((B, H_kv, L, d))
    v = rng.standard_normal((B, H_kv, L, d))
    beta = rng.uniform(-3, 3, H_q)
    M0 = rng.standard_normal((B, H_kv, d, d))
    z0 = rng.uniform(0.5, 2.0, (B, H_kv, d))
    return q, k, v, beta, M0, z0, S


def _sp_worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, beta, M0, z0, S = _sp_problem()
        L = q.shape[2]
        l0, l1 = shard.segment_range(L, S, world, rank)
        t = torch.from_numpy
        out, M_T, z_T = shard.sequence_parallel_forward(
            t(q[:, :, l0:l1].copy()), t(k[:, :, l0:l1].copy()), t(v[:, :, l0:l1].copy()), t(beta),
            t(M0), t(z0), S, forward=_oracle_forward, state_update=_oracle_state_update,
            state_sum=_host_state_sum)
        ref_out, ref_M, ref_z = oracle.infini_attention_forward(q, k, v, beta, M0, z0, S, "linear")
        results[rank] = ((l0, l1),
                         float(np.max(np.abs(out.numpy() - ref_out[:, :, l0:l1]), initial=0.0)),
                         float(np.max(np.abs(M_T.numpy() - ref_M))),
                         float(np.max(np.abs(z_T.numpy() - ref_z))))
    finally:
        dist.destroy_process_group()


def test_segment_range_partition():
    for L, S in ((100, 16), (64, 64), (1, 5), (1000, 128), (2048, 1)):
        T = -(-L // S)
        for world in (1, 2, 3, 4, 8):
            rs = [shard.segment_range(L, S, world, r) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == L
            assert all(rs[i][1] == rs[i + 1][0] for i in range(world - 1))
            # whole segments: every cut sits on a segment boundary
            assert all(a % S == 0 for a, _ in rs if a < L)
            counts = [-(-(b - a) // S) for a, b in rs]
            assert sum(counts) == T and max(counts) - min(counts) <= 1


def test_prefix_states_in_rank_order():
    M0 = torch.full((1, 1, 2, 2), 1.0, dtype=torch.float64)
    z0 = torch.full((1, 1, 2), 2.0, dtype=torch.float64)
    ups = torch.stack([torch.cat([torch.full((4,), float(10 ** r)), torch.full((2,), float(r))])
                       for r in range(3)]).double()
    M_in, z_in, M_T, z_T = shard.prefix_states(ups, 2, M0, z0, _host_state_sum)
    assert torch.all(M_in == 12.0) and torch.all(z_in == 3.0)
    assert torch.all(M_T == 112.0) and torch.all(z_T == 5.0)
    M_in, z_in, _, _ = shard.prefix_states(ups, 0, M0, z0, _host_state_sum)
    assert torch.equal(M_in, M0) and torch.equal(z_in, z0)


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_parallel_linear_rule_gloo(world):
    """Sequence cut into per-rank runs of whole segments, one all-gather of
    the runs' state updates, exclusive prefix, then each rank's own forward:
    the rank's rows of `out` and the final state equal the single-process
    forward (float64 oracle as the per-rank compute)."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    mp.start_processes(_sp_worker, args=(world, port, results), nprocs=world, join=True,
                       start_method="spawn")
    assert sorted(results.keys()) == list(range(world))
    covered = 0
    for r in range(world):
        (l0, l1), e_out, e_M, e_z = results[r]
        assert l0 == covered
        covered = l1
        assert e_out <= 1e-12 and e_M <= 1e-12 and e_z <= 1e-12, (r, e_out, e_M, e_z)
    assert covered == 100
