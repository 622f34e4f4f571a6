"""The multi-rank benchmark path on CPU: two gloo ranks, each with its own replica of a workload
(weak scaling), no data-path collective; only the timing is reduced (max over ranks)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import kda_workloads as W
import oracle


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}")
    try:
        assert bench.dist_env()[:2] == (rank, world)
        # every rank solves its own replica (distinct seed), on the oracle here (no GPU)
        w = W.make("tiny_fp32_T64_d16", seed=bench.rank_seed("tiny_fp32_T64_d16", rank))
        o, _ = oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens,
                                  w.state_pool, w.state_indices)
        local_ms = 10.0 + 5.0 * rank
        ms = bench.max_over_ranks(local_ms, dist)
        value = bench.whole_job_throughput(w.total_tokens, world, ms)
        out[rank] = (ms, value, float(np.abs(o).sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_by_the_slowest_and_work_on_distinct_replicas():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    (ms0, v0, s0), (ms1, v1, s1) = out[0], out[1]
    assert ms0 == ms1 == 15.0                       # the slower rank's time on every rank
    assert v0 == v1 == pytest.approx(64 * 2 / 0.015)  # units of both ranks over that time
    assert s0 != s1                                 # each rank had its own inputs


def test_rank_seeds_are_distinct():
    seeds = {bench.rank_seed("long_T131072_H32_cp16", r) for r in range(8)}
    assert len(seeds) == 8


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        workload = "tiny_fp32_T64_d16"
        steps = 1
        warmup = 0
        ref_step_seconds = 0.01

    assert bench.run_reference(Args()) == 0  # returns at once, prints nothing
