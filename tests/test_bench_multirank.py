"""World-size-2 checks of the benchmark's multi-rank host logic on CPU (gloo): each
rank draws its own batch, the job time is the slowest rank's, and the whole-job rate
counts every rank's work.  No GPU is used."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, local_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(local_ms[rank], dist, "cpu")
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(rank))
        out[rank] = (ms, seeds)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_distinct_batches():
    world, port = 2, _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    local_ms = [3.5, 4.25]
    mp.start_processes(_worker, args=(world, port, local_ms, out), nprocs=world, start_method="spawn", join=True)
    for rank in range(world):
        ms, seeds = out[rank]
        assert ms == max(local_ms)
        assert len(set(seeds)) == world


def test_whole_job_rate_counts_every_rank():
    one = bench.whole_job_rate(9.27e12, 10, 1, 20.0)
    two = bench.whole_job_rate(9.27e12, 10, 2, 20.0)
    assert two == pytest.approx(2 * one)
    assert one == pytest.approx(9.27e12 * 10 / 0.02 / 1e12)


def test_algorithmic_bytes_of_a_gemm_and_a_quantiser():
    """MXFP4 operands: half a byte per element plus one scale byte per 32; D in BF16."""
    M, N, K = 32760, 13824, 5120
    assert bench.gemm_bytes(M, N, K) == pytest.approx(M * K * 0.53125 + N * K * 0.53125 + 2 * M * N)
    assert bench.gemm_bytes(M, N, K, 1.0) == pytest.approx(M * K + N * K * 0.53125 + 2 * M * N)  # FP8 A
    assert bench.gemm_bytes(M, N, K) / 1e6 == pytest.approx(1032.0, abs=0.5)  # Wan FFN up: A + B + D


def test_weight_rotation_for_small_working_sets():
    l2 = 126 << 20
    w = 13824 * 5120 * 17 // 32  # 37.6 MB of packed weights
    assert bench.weight_copies("m_sweep", 50 << 20, w, l2) == 8  # >= 2 x L2 in total
    assert bench.weight_copies("m_sweep", 50 << 20, 200 << 20, l2) == 4  # at least 4
    assert bench.weight_copies("m_sweep", 5 * l2, w, l2) == 1  # working set beyond 4 x L2
    assert bench.weight_copies("flux_w4a8", 50 << 20, w, l2) == 1  # other workloads flush instead
