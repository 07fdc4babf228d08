"""The multi-GPU path is replicas only (no exchange step): world-size-2 checks of the benchmark's
cross-rank logic on CPU with the gloo backend -- the max-over-ranks timing reduction every rank
takes part in, the per-replica step time and the whole-job throughput taken from it, and the
reference arm's rank-0-only rule."""
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


def _worker(rank: int, world: int, port: int, out):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ms = [12.5, 17.25][rank]                     # each replica's own timed-region length
        m = bench.max_over_ranks(ms, world)
        out[rank] = (m, bench.per_replica_us_per_step(m, 10), bench.aggregate_steps_per_s(m, 10, world))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_with_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        m, per_step, agg = res[rank]
        assert m == 17.25                            # the slowest rank's time, on every rank
        assert per_step == pytest.approx(17.25e3 / 10)    # a replica's step latency
        assert agg == pytest.approx(10 * 2 / 17.25e-3)    # decode steps per second, whole job


def test_single_rank_reduction_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.per_replica_us_per_step(2.0, 4) == 500.0
    assert bench.aggregate_steps_per_s(2.0, 4, 1) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), {"workload": "tiny-2k", "window": 0, "gamma": 3, "steps": 1, "warmup": 0})()
    bench.run_reference(args)                        # returns at once: no work, no output
    assert capsys.readouterr().out == ""
