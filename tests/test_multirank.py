"""Multi-rank host logic of the benchmark on CPU with gloo, world size 2:
the timing reduction takes the slowest rank, the whole-job value counts
every rank's shard, per-rank inputs differ only in their values, and the
reference arm runs on rank 0 alone."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist

    import bench
    from workloads import config_tiny, fill_values_torch

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports elapsed times (10 + r, 3 - r): the max is taken per element
        got = bench.max_over_ranks([10.0 + rank, 3.0 - rank])
        L = config_tiny()
        V = fill_values_torch(L, "cpu", value_seed=L.seed + 7 * rank)
        digest = float(V.q.float().sum())
        digests = [None] * world
        dist.all_gather_object(digests, (L.num_seqs, L.total_blocks_touched(), digest))
        out[rank] = (got, digests)
    finally:
        dist.destroy_process_group()


def test_timing_reduction_and_shards_with_two_gloo_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        got, digests = out[rank]
        assert got == [11.0, 3.0]
        # same shard shape on every rank, different values
        assert digests[0][:2] == digests[1][:2]
        assert digests[0][2] != digests[1][2]


def test_whole_job_value_counts_every_rank():
    import bench

    one = bench.whole_job_gbs(1, 1_000_000_000, 1.0)
    assert one == pytest.approx(1000.0)
    assert bench.whole_job_gbs(4, 1_000_000_000, 1.0) == pytest.approx(4 * one)


def test_reference_arm_runs_on_rank_zero_only(capsys, monkeypatch):
    import bench

    monkeypatch.setenv("RANK", "1")
    rc = bench.run_reference(bench.parse_args(["--impl", "reference", "--gpus", "2", "--steps", "1",
                                               "--warmup", "0", "--config", "tiny"]))
    assert rc == 0
    assert capsys.readouterr().out == ""


def _split_rank_main(rank, world, port, out):
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from paged_kv_cache_357_b200.split import gather_partials
    from workloads import fill_values_numpy, random_layout

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L = random_layout(31, [5, 40, 64, 100, 0], dtype="bf16", block_size=8, num_q_heads=4, num_kv_heads=2,
                          head_dim=16, write_new_token=False)
        V = fill_values_numpy(L)
        # rank r holds tokens [32 r, 32 (r + 1)) of every sequence (the last rank the rest)
        a = 32 * rank
        b = 32 * (rank + 1) if rank < world - 1 else 1 << 20
        lens = np.clip(L.seq_lens - a, 0, b - a).astype(np.int32)
        tables = np.zeros_like(L.block_tables)
        tables[:, : L.block_tables.shape[1] - a // 8] = L.block_tables[:, a // 8:]
        part, lse = oracle.decode_lse(V.q, V.k_pool, V.v_pool, tables, lens, L.scale, L.num_kv_heads, L.dtype)
        outs, lses = gather_partials(torch.from_numpy(part), torch.from_numpy(lse))
        merged, merged_lse = oracle.merge_outputs(outs.numpy(), lses.numpy())
        full, full_lse = oracle.decode_lse(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale,
                                           L.num_kv_heads, L.dtype)
        fin = np.isfinite(full_lse)
        out[rank] = (float(np.abs(merged - full).max()), float(np.abs(merged_lse[fin] - full_lse[fin]).max()),
                     bool(np.array_equal(np.isinf(merged_lse), np.isinf(full_lse))), tuple(outs.shape))
    finally:
        dist.destroy_process_group()


def test_split_sequence_partials_gathered_and_merged_with_two_gloo_ranks():
    """Two ranks each hold a block range of every sequence: their partial
    decodes (the oracle's, on CPU) gathered by split.gather_partials and
    merged equal the whole decode on both ranks."""
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_split_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        err, lse_err, same_inf, shape = out[rank]
        assert shape == (world, 5, 4, 16)
        assert err < 1e-12 and lse_err < 1e-12 and same_inf
