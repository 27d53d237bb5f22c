"""The benchmark's multi-rank host logic on CPU: two gloo ranks reduce their timed totals to the
max over ranks, rank 0 derives whole-job throughput from it, and the reference arm's non-zero
ranks exit without work. (The path itself has no collective: replicas only.)"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_total_ms = [100.0, 250.0][rank]
        t = bench.reduce_max(my_total_ms, world, "cpu")
        v = bench.throughput(1e12, 10, world, t)
        out[rank] = (t, v)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, start_method="spawn")
    for r in (0, 1):
        t, v = out[r]
        assert t == 250.0                              # slowest rank decides
        assert v == pytest.approx(1e12 * 10 * 2 / 0.25 / 1e12)


def test_reference_arm_nonzero_rank_exits_without_work(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"]) == 0


def test_throughput_single_rank():
    assert bench.throughput(824.6e9, 10, 1, 5000.0) == pytest.approx(824.6e9 * 10 / 5.0 / 1e12)
    nums = bench.workload_numbers(__import__("optimizer_fp8_cast_b200.synth", fromlist=["x"]).LINEAR4096)
    assert 3 * sum(nums["gemm_flop"]) == 824_633_720_832
    assert nums["h2d"] == nums["d2h"] == 134_217_728
