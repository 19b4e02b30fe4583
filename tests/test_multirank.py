"""The multi-GPU host path of bench.py on CPU: two gloo ranks, the same helpers the NCCL run uses.

Each rank processes its own sequence (seed + 7919 r, no collective on the data path); the job's
time is the slowest rank's and its throughput counts every rank's tokens.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench
    from cross_model_attention_mr_b200.workloads import config, draw_layers, shrink
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        spec = bench.rank_spec(shrink(config(4), L=256, H_s=2, H_r=2), rank)
        lay = draw_layers(spec)[0]
        sig = torch.tensor([float(np.float64(lay.Q.astype(np.float64).sum()))], dtype=torch.float64)
        sigs = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sigs, sig)
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, "cpu")
        value = bench.job_tokens_per_s(world, spec.L, ms)
        all_fine = bench.all_ranks_ok(True, dist, "cpu")
        one_failed = bench.all_ranks_ok(rank != 1, dist, "cpu")  # rank 1 reports a device error
        out[rank] = (spec.seed, [float(x.item()) for x in sigs], ms, value, all_fine, one_failed)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_independent_sequences_and_max_time():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    seeds = [out[r][0] for r in range(world)]
    assert seeds[1] == seeds[0] + 7919
    sigs = out[0][1]
    assert sigs == out[1][1] and sigs[0] != sigs[1]  # different sequences, seen alike by both ranks
    for r in range(world):
        _, _, ms, value, all_fine, one_failed = out[r]
        assert ms == pytest.approx(15.0)  # the slowest rank's time on every rank
        assert value == pytest.approx(world * 256 / 15e-3)
        assert all_fine and not one_failed  # every rank takes the error path together


def test_single_rank_helpers_without_a_process_group():
    sys.path.insert(0, ROOT)
    import bench
    from cross_model_attention_mr_b200.workloads import config
    spec = config(4)
    assert bench.rank_spec(spec, 0) is spec
    assert bench.max_over_ranks(12.5, None, "cpu") == 12.5
    assert bench.job_tokens_per_s(1, 32768, 100.0) == pytest.approx(327680.0)
    assert bench.all_ranks_ok(False, None, "cpu") is False
