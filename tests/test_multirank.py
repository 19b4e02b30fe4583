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


def _synthetic_map(mr, nnz, capacity, seed, dtype=None):
    """A compressed map with seeded contents (the transfer moves bytes; it computes nothing)."""
    g = torch.Generator().manual_seed(seed)
    dtype = mr.MR_BF16 if dtype is None else dtype
    m = mr.Map(3, 512, 64, dtype, capacity, "cpu")
    n = min(nnz, capacity)
    m.row_ptr.copy_(torch.cumsum(torch.randint(0, 3, (m.row_ptr.numel(),), generator=g), 0).to(torch.int32))
    m.kept_bits.copy_(torch.randint(-2**31, 2**31 - 1, m.kept_bits.shape, generator=g, dtype=torch.int64).to(torch.int32))
    m.kept_mass.copy_(torch.rand(m.kept_mass.shape, generator=g))
    m.col_idx[:n].copy_(torch.randint(0, 8, (n,), generator=g, dtype=torch.int32))
    if dtype == mr.MR_FP8_E4M3:
        m.vals[:n].copy_(torch.randint(0, 127, (n, 64, 64), generator=g, dtype=torch.int32).to(torch.uint8))
        m.tile_scale[:n].copy_(torch.rand((n, mr.fp8_scales_per_tile(64)), generator=g))
    else:
        m.vals[:n].copy_(torch.randn((n, 64, 64), generator=g).to(torch.bfloat16))
    m.nnz.fill_(nnz)
    return m


def test_map_copy_between_devices_keeps_every_array():
    """Map.to: the copy a receiving rank makes to move a received map onto its GPU (here host to
    host) keeps capacity, flags and every array bit for bit."""
    from cross_model_attention_mr_b200 import mr
    for dt in (None, mr.MR_FP8_E4M3):
        src = _synthetic_map(mr, 29, 32, seed=7, dtype=dt)
        dst = src.to("cpu")
        assert dst is not src and dst.capacity == src.capacity and dst.c.capacity_tiles == src.c.capacity_tiles
        assert dst.dtype == src.dtype and dst.c.renormalised == src.c.renormalised
        for name in ("row_ptr", "col_idx", "vals", "kept_mass", "kept_bits", "nnz", "tile_scale"):
            a, b = getattr(src, name), getattr(dst, name)
            assert (a is None) == (b is None)
            if a is not None:
                assert a.data_ptr() != b.data_ptr() and torch.equal(a, b), name


def _map_rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    from cross_model_attention_mr_b200 import mr
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        results = []
        for case, (nnz, cap, dt) in enumerate([(37, 40, None), (50, 40, None), (0, 16, None),
                                               (29, 32, mr.MR_FP8_E4M3)]):
            local = _synthetic_map(mr, nnz, cap, seed=100 + case, dtype=dt)
            if rank == 0:
                mr.send_map(local, 1)
                continue
            got = mr.recv_map(0, device="cpu")
            n = min(nnz, cap)
            same = (got.capacity == n and int(got.nnz.item()) == nnz and got.c.capacity_tiles == n
                    and torch.equal(got.row_ptr, local.row_ptr) and torch.equal(got.kept_bits, local.kept_bits)
                    and torch.equal(got.kept_mass, local.kept_mass)
                    and torch.equal(got.col_idx[:n], local.col_idx[:n])
                    and torch.equal(got.vals[:n], local.vals[:n])
                    and (local.tile_scale is None or torch.equal(got.tile_scale[:n], local.tile_scale[:n])))
            results.append(bool(same))
        out[rank] = results
    finally:
        dist.destroy_process_group()


def test_compressed_map_moves_between_gloo_ranks_bit_exactly():
    """send_map / recv_map: a map, an overflowed map (kept tiles beyond capacity stay unstored on the
    receiver), an empty one and an fp8 map with its scales arrive bit-exactly."""
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_map_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert out[1] == [True, True, True, True]


# ------------------------------------------------------------------------------------------------
# One sequence split across ranks by query-block range: partition, K/V shard exchange, and the
# independence of the per-rank work (the oracle on each rank's units equals the single-rank run).
# ------------------------------------------------------------------------------------------------
def test_split_ranges_cover_every_query_block_once():
    from cross_model_attention_mr_b200 import mr
    for nqb, world, align in [(256, 2, 1), (256, 8, 1), (64, 4, 2), (128, 3, 2), (3, 4, 1)]:
        ranges = mr.split_query_blocks(nqb, world, align)
        assert len(ranges) == world and ranges[0][0] == 0 and ranges[-1][1] == nqb
        for (a, b), (c, _) in zip(ranges[:-1], ranges[1:]):
            assert a <= b == c                                # contiguous, in order, disjoint
        assert all(b % align == 0 or b == nqb for _, b in ranges)
        if nqb >= 4 * world * align:                          # balanced by causal work
            work = [sum(I + 1 for I in range(a, b)) for a, b in ranges]
            assert max(work) <= 1.25 * (nqb * (nqb + 1) / 2) / world


def _split_rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import oracle
    from cross_model_attention_mr_b200 import mr
    from cross_model_attention_mr_b200.workloads import config, draw_layers, shrink
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        spec = shrink(config(4), L=1024, H_s=2, H_r=2)
        lay = draw_layers(spec)[0]
        nqb = spec.L // spec.block
        ranges = mr.split_query_blocks(nqb, world)
        shards = mr.row_shards(spec.L, ranges, spec.block)
        b, e = shards[rank]
        # this rank only holds its own rows of K and V; the all-gather rebuilds the sequence
        K_full = mr.gather_row_shards(torch.from_numpy(lay.K[:, b:e].copy()), shards)
        V_full = mr.gather_row_shards(torch.from_numpy(lay.V[:, b:e].copy()), shards)
        q0, q1 = ranges[rank]
        units = [h * nqb + I for h in range(spec.H_s) for I in range(q0, q1)]
        r = oracle.compress(lay.Q, K_full.numpy(), spec.scale, float(np.float32(spec.p)), spec.block, lay.bias,
                            units=units)
        rows = np.arange(b, e, 37)
        O = oracle.retrieve_rows(lay.Q, K_full.numpy(), spec.scale, spec.block, r.kept, lay.W, V_full.numpy(),
                                 rows, lay.bias)
        out[rank] = (bool(np.array_equal(K_full.numpy(), lay.K)), bool(np.array_equal(V_full.numpy(), lay.V)),
                     (q0, q1), r.kept[:, q0:q1].copy(), rows, O)
    finally:
        dist.destroy_process_group()


def test_split_sequence_two_gloo_ranks_match_one_rank():
    import oracle
    from cross_model_attention_mr_b200.workloads import config, draw_layers, shrink
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_split_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    spec = shrink(config(4), L=1024, H_s=2, H_r=2)
    lay = draw_layers(spec)[0]
    full = oracle.compress(lay.Q, lay.K, spec.scale, float(np.float32(spec.p)), spec.block, lay.bias)
    covered = []
    for rk in range(world):
        k_ok, v_ok, (q0, q1), kept, rows, O = out[rk]
        assert k_ok and v_ok                                   # the gathered K and V are the sequence's
        assert np.array_equal(kept, full.kept[:, q0:q1])       # the rank's selection is the full run's
        want = oracle.retrieve_rows(lay.Q, lay.K, spec.scale, spec.block, full.kept, lay.W, lay.V, rows, lay.bias)
        assert np.max(np.abs(O - want)) < 1e-12
        covered += list(range(q0, q1))
    assert covered == list(range(spec.L // spec.block))
