"""Compress on one rank, retrieve on another (MapFlow section 6: the sender's compressed
block-sparse maps are transferred to the receiver, which runs the fused retrieval locally).

Two processes on the one GPU this test gets, connected by gloo: rank 0 compresses a layer on the
GPU and sends the map through `send_map` as host tensors; rank 1 receives it with `recv_map`,
moves it onto the GPU, retrieves with its own W and V, and checks every sampled row against the
fp64 oracle on the received kept sets.  The two ranks' kernels never wait on each other: the only
exchange is the host-side transfer between the two launches.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, map_dtype, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import oracle
    from cross_model_attention_mr_b200 import mr
    from cross_model_attention_mr_b200.workloads import config, draw_layers, shrink
    from parity import OUT_TOL, dev, p32
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        spec = shrink(config(4), L=1024, H_s=4, H_r=6)
        lay = draw_layers(spec)[0]
        dt = mr.MR_BF16 if map_dtype == "bf16" else mr.MR_FP8_E4M3
        if rank == 0:
            m = mr.compress(dev(lay.Q, "bf16"), dev(lay.K, "bf16"), p32(spec.p), spec.block,
                            bias=mr.Bias.from_spec(lay.bias), scale=spec.scale, map_dtype=dt)
            st = m.ws.sync_status()
            mr.send_map(m.to("cpu"), 1)
            out[0] = (st, m.nnz_host())
        else:
            got = mr.recv_map(0, device="cpu").to("cuda")
            ws = mr.Workspace(mr.retrieve_workspace_bytes(got, spec.H_r, spec.d_v, 1))
            O = mr.retrieve(got, torch.from_numpy(lay.W).cuda(), dev(lay.V, "bf16"), ws=ws)
            st = ws.sync_status()
            rows = np.arange(0, spec.L, 29)
            want = oracle.retrieve_rows(lay.Q, lay.K, spec.scale, spec.block, got.kept_bits_host(), lay.W, lay.V,
                                        rows, lay.bias)
            err = float(np.max(np.abs(O[:, :, rows].float().cpu().numpy() - want)))
            out[1] = (st, got.nnz_host(), err, OUT_TOL[map_dtype] * float(np.abs(lay.V).max()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("map_dtype", ["bf16", "fp8"])
def test_map_compressed_on_one_rank_retrieved_on_another(map_dtype):
    assert torch.cuda.is_available()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(2, _free_port(), map_dtype, out), nprocs=2, start_method="spawn")
    st0, nnz0 = out[0]
    st1, nnz1, err, tol = out[1]
    assert st0 == 0 and st1 == 0
    assert nnz0 == nnz1 > 0
    assert err <= tol, (err, tol)
