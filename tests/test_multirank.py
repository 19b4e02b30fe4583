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
    # the other workloads' lines: tokens per step (config 5: every request's prefix and suffix)
    assert bench.config_tokens_per_step(config(2)) == 4096
    assert bench.config_tokens_per_step(config(5), [512, 2048, 1000]) == 3 * 4096 + 3560


def _synthetic_map(mr, nnz, capacity, seed):
    """A compressed map with seeded contents (the transfer moves bytes; it computes nothing)."""
    g = torch.Generator().manual_seed(seed)
    m = mr.Map(3, 512, 64, mr.MR_BF16, capacity, "cpu")
    n = min(nnz, capacity)
    m.row_ptr.copy_(torch.cumsum(torch.randint(0, 3, (m.row_ptr.numel(),), generator=g), 0).to(torch.int32))
    m.kept_bits.copy_(torch.randint(-2**31, 2**31 - 1, m.kept_bits.shape, generator=g, dtype=torch.int64).to(torch.int32))
    m.kept_mass.copy_(torch.rand(m.kept_mass.shape, generator=g))
    m.col_idx[:n].copy_(torch.randint(0, 8, (n,), generator=g, dtype=torch.int32))
    m.vals[:n].copy_(torch.randn((n, 64, 64), generator=g).to(torch.bfloat16))
    m.nnz.fill_(nnz)
    return m


def _map_rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    from cross_model_attention_mr_b200 import mr
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        results = []
        for case, (nnz, cap) in enumerate([(37, 40), (50, 40), (0, 16)]):
            local = _synthetic_map(mr, nnz, cap, seed=100 + case)
            if rank == 0:
                mr.send_map(local, 1)
                continue
            got = mr.recv_map(0, device="cpu")
            n = min(nnz, cap)
            same = (got.capacity == n and int(got.nnz.item()) == nnz and got.c.capacity_tiles == n
                    and torch.equal(got.row_ptr, local.row_ptr) and torch.equal(got.kept_bits, local.kept_bits)
                    and torch.equal(got.kept_mass, local.kept_mass)
                    and torch.equal(got.col_idx[:n], local.col_idx[:n])
                    and torch.equal(got.vals[:n].view(torch.int16), local.vals[:n].view(torch.int16)))
            results.append(bool(same))
        out[rank] = results
    finally:
        dist.destroy_process_group()


def test_compressed_map_moves_between_gloo_ranks_bit_exactly():
    """send_map / recv_map: a map, an overflowed map (kept tiles beyond capacity stay unstored on the
    receiver) and an empty one arrive bit-exactly."""
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_map_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert out[1] == [True, True, True]
