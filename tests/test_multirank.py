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
